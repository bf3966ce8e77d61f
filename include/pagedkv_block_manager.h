/*
 * pagedkv_block_manager.h -- host-side manager of the paged KV-cache pool
 * (part of libpagedkv.so; plain C ABI, host memory only, no CUDA calls).
 *
 * What it does follows the vLLM pages:
 *   - case-study page "vLLM 与 PagedAttention", section 二 "PagedAttention 的解法":
 *     the KV cache of a request is cut into fixed-size blocks taken from one
 *     shared pool only when needed (the 7th block is taken when generation
 *     reaches the 100th token); a per-request block table maps logical to
 *     physical blocks; requests with a common prefix point at the same physical
 *     blocks and copy on write;
 *   - same page, section 四 "Prefix Caching": the first request's prefix KV is
 *     kept in an LRU cache and later requests with the same prefix reuse it and
 *     skip its prefill;
 *   - 298.name page, "PagedKVCache" sketch: allocate ceil(seq_len / block_size)
 *     pages for a request and record them in its page table;
 *   - guide page "指南", "Copy-on-Write": shared blocks are read-only until a
 *     request diverges, then copied.
 *
 * Policy (deterministic, so that a plain model can reproduce it exactly):
 *   - Free blocks form a stack; the pool starts as [0, 1, ..., N-1] with block
 *     0 on top.  A freed block that is not cached is pushed on top.
 *   - With prefix caching on, every FULL block is identified by a hash of its
 *     parent block's hash and its block_size token ids; the cache maps hash ->
 *     block.  A cached block whose reference count drops to 0 stays cached and
 *     joins the tail of the LRU list; a cache hit takes it back out.
 *   - A new block comes from the free stack, else by evicting the head of the
 *     LRU list (its cache entry is dropped).  No block left -> PKV_BM_ENOSPACE.
 *   - Appending a token to a sequence whose last block is shared (reference
 *     count > 1) first copies that block: the manager takes a new block, reports
 *     the (src, dst) pair for pkv_copy_blocks, and repoints the table.
 *   - A block that becomes full gets its hash; it enters the cache if no block
 *     with that hash is cached yet.
 *   - Freeing a sequence releases its blocks from the last to the first, so a
 *     cached prefix's deeper blocks enter the LRU list (and leave it) first.
 *   - Swapping (case-study page, section 三: under memory pressure a request is
 *     pre-empted by moving its KV to CPU memory, and resumed later; tutorial
 *     page 4.3).  An optional host pool of num_host_blocks blocks has its own
 *     free stack (block 0 on top) and a reference count per host block.
 *     Swapping out a group of sequences (one, or e.g. the samples of one
 *     request, which share blocks) takes one host block per DISTINCT device
 *     block of the group's tables, in order of first appearance (sequences in
 *     the given order, positions in logical order), from the top of that
 *     stack; reports those (device, host) pairs; points every table entry at
 *     its block's host copy; then releases each sequence's device blocks like
 *     a free (sequences in order, each last to first; cached ones stay
 *     cached).  Swapping a group in takes one device block per distinct host
 *     block, in order of first appearance (free stack, else LRU eviction),
 *     reports the (host, device) pairs, points the tables at them (a block
 *     shared by k tables gets reference count k), and drops the sequences'
 *     host references (sequences in order, each last to first); a host block
 *     left with none goes back on top of the host stack.  Swapped-in blocks
 *     are private to the group: they are not re-entered in the prefix cache
 *     (the hash chain of later blocks continues).  A swapped-out sequence can
 *     only be swapped in, freed (dropping its host references) or asked for
 *     its token count.
 *
 * The manager is not thread-safe; one owner calls it.
 */
#ifndef PAGEDKV_BLOCK_MANAGER_H
#define PAGEDKV_BLOCK_MANAGER_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pkv_block_manager pkv_block_manager;

enum {
    PKV_BM_OK = 0,
    PKV_BM_EINVAL = -1,    /* bad argument, unknown or duplicate sequence id */
    PKV_BM_ENOSPACE = -6,  /* the pool has no free or evictable block left */
    PKV_BM_EBUFFER = -7    /* an output buffer is too small */
};

/* New manager over a pool of num_blocks blocks of block_size tokens.
 * prefix_caching != 0 enables the hash-chain prefix cache.  NULL on bad input. */
pkv_block_manager* pkv_bm_create(int64_t num_blocks, int block_size, int prefix_caching);
void pkv_bm_destroy(pkv_block_manager* bm);

/* Register sequence seq_id with its prompt token ids (num_tokens >= 0) and take
 * the blocks that hold them.  With prefix caching, full blocks whose hash chain
 * is cached are shared instead; *num_cached_tokens receives how many leading
 * tokens are already in the cache (a multiple of block_size; their prefill can
 * be skipped).  On failure nothing changes. */
int pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq_id, const int32_t* tokens, int64_t num_tokens,
                        int64_t* num_cached_tokens);

/* Append num_tokens tokens to seq_id.  slots_out[i] receives the physical slot
 * (block * block_size + offset) of the i-th appended token.  Copy-on-write
 * pairs go to cow_pairs_out ([max_pairs][2] int64, (src, dst)), their count to
 * *num_pairs; run them (pkv_copy_blocks) before writing the new tokens' K/V.
 * On failure nothing changes. */
int pkv_bm_append(pkv_block_manager* bm, int64_t seq_id, const int32_t* tokens, int64_t num_tokens,
                  int64_t* slots_out, int64_t* cow_pairs_out, int64_t max_pairs, int64_t* num_pairs);

/* One decode step for a batch: append tokens[i] to seq_ids[i] for i < n.
 * slots_out[i] receives its slot; the copy-on-write pairs of the whole batch
 * go to cow_pairs_out ([max_pairs][2]), their count to *num_pairs.  The
 * sequences are processed in order; on failure the ones before the failing
 * index stay appended and *num_done tells how many. */
int pkv_bm_append_batch(pkv_block_manager* bm, const int64_t* seq_ids, const int32_t* tokens, int64_t n,
                        int64_t* slots_out, int64_t* cow_pairs_out, int64_t max_pairs, int64_t* num_pairs,
                        int64_t* num_done);

/* child shares every block of parent (parallel sampling / beam search).
 * append, fork (as parent), slots and block_table reject a swapped-out
 * sequence with PKV_BM_EINVAL. */
int pkv_bm_fork(pkv_block_manager* bm, int64_t parent_id, int64_t child_id);

/* Release seq_id's blocks (cached ones stay cached until evicted). */
int pkv_bm_free(pkv_block_manager* bm, int64_t seq_id);

/* Physical slots of positions [start, start + count) of seq_id. */
int pkv_bm_slots(const pkv_block_manager* bm, int64_t seq_id, int64_t start, int64_t count, int64_t* slots_out);

/* seq_id's block table into out[0 .. max_blocks) (unused entries -1); the
 * number of blocks goes to *num_blocks. */
int pkv_bm_block_table(const pkv_block_manager* bm, int64_t seq_id, int32_t* out, int64_t max_blocks,
                       int64_t* num_blocks);

/* Tokens held by seq_id, or a negative status. */
int64_t pkv_bm_num_tokens(const pkv_block_manager* bm, int64_t seq_id);

/* Counters: [0] free blocks, [1] evictable cached blocks, [2] cached blocks
 * in total, [3] cache-hit blocks so far, [4] evictions so far, [5] CoW copies
 * so far, [6] sequences (resident and swapped out), [7] free host blocks,
 * [8] swapped-out sequences.  Returns the number written (<= n). */
int pkv_bm_stats(const pkv_block_manager* bm, int64_t* out, int n);

/* Size the host pool used by swapping (0 at creation).  Allowed only while no
 * sequence is swapped out; the host free stack restarts as [0, ..., n-1]. */
int pkv_bm_set_host_blocks(pkv_block_manager* bm, int64_t num_host_blocks);

/* Pre-empt seq_id: pairs_out ([max_pairs][2] int64) receives one (device
 * block, host block) pair per block of its table, in logical order, and
 * *num_pairs their count.  Copy those blocks device -> host (pkv_swap_blocks)
 * before any later call can hand the released device blocks out again, i.e.
 * enqueue the copy before the K/V writes of the next step.  PKV_BM_ENOSPACE
 * when the host pool has too few free blocks, PKV_BM_EBUFFER when max_pairs is
 * too small; on failure nothing changes. */
int pkv_bm_swap_out(pkv_block_manager* bm, int64_t seq_id, int64_t* pairs_out, int64_t max_pairs,
                    int64_t* num_pairs);

/* Resume a swapped-out seq_id: pairs_out receives one (host block, device
 * block) pair per block, in logical order; copy them host -> device before the
 * sequence's next attention.  The sequence's table then lists the new device
 * blocks.  The host blocks named as sources go back to the host free stack at
 * once, so a later pkv_bm_swap_out (of this step or a later one) may name one
 * of them as its copy target: enqueue this call's host -> device copies before
 * the device -> host copies of any later swap-out, on the same stream (or with
 * an event between the two streams).  PKV_BM_ENOSPACE when the device pool has too few free or evictable
 * blocks, PKV_BM_EBUFFER when max_pairs is too small; on failure nothing
 * changes. */
int pkv_bm_swap_in(pkv_block_manager* bm, int64_t seq_id, int64_t* pairs_out, int64_t max_pairs,
                   int64_t* num_pairs);

/* The same for n >= 1 distinct sequences at once: blocks they share cross to
 * the host once and are shared again after swap-in (pairs: one per distinct
 * block, see the policy above).  pkv_bm_swap_out / pkv_bm_swap_in are the
 * one-sequence case.  PKV_BM_EINVAL if an id is unknown, repeated, or not
 * resident (out) / not swapped out (in). */
int pkv_bm_swap_out_group(pkv_block_manager* bm, const int64_t* seq_ids, int64_t n, int64_t* pairs_out,
                          int64_t max_pairs, int64_t* num_pairs);
int pkv_bm_swap_in_group(pkv_block_manager* bm, const int64_t* seq_ids, int64_t n, int64_t* pairs_out,
                         int64_t max_pairs, int64_t* num_pairs);

/* Reference count of a physical block (or a negative status). */
int pkv_bm_ref_count(const pkv_block_manager* bm, int64_t block);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_BLOCK_MANAGER_H */
