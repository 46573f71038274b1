/*
 * pa_kv_manager.h -- C ABI of the host-side KV-cache block manager.
 *
 * What it does.  It owns the bookkeeping of one KV pool of `num_blocks`
 * physical blocks of `block_size` token slots: which physical blocks each
 * sequence's logical blocks map to (its block table), how many tables
 * reference each block, and which unreferenced blocks still hold a cached full
 * block.  Its outputs are exactly the inputs of the device calls in pa.h: the
 * slot of every new token (pa_reshape_and_cache's slot_mapping), the (src, dst)
 * pairs to copy before writing (pa_copy_blocks), and the block tables and
 * context lengths of a batch (pa_decode, pa_chunked_prefill).  It runs on the
 * host and touches no device memory.
 *
 * Sources, by page title and section:
 *   "vLLM 基本原理", PagedAttention: logical blocks, physical blocks and the
 *     block table; on-demand allocation (a new physical block only when the
 *     current one is full, so only a sequence's last block may be partly used);
 *     memory sharing (outputs of one prompt point at the same prompt blocks and
 *     get private blocks only for their own new tokens).
 *   "当大模型推理遇上内存瓶颈", 2.2 (a reference count per block drives
 *     copy-on-write), 2.3 (sharing a whole sequence, its first n blocks --
 *     share_prefix -- or chosen logical blocks -- share_blocks), 3.3 (with
 *     reference counts only the first writer of a shared block copies it).
 *   "vLLM 定位与核心机制详解", 六.1 (a finished sequence's blocks are freed at
 *     once) and 六.3 (prefix caching: a full block is identified by its tokens
 *     from position 0; a new request reuses the cached blocks of its identical
 *     prefix, whole blocks only).
 *
 * Rules where the pages leave a choice:
 *   - A fresh block is the lowest-numbered free block that never held a cached
 *     block; when there is none, the cached block that became unreferenced
 *     longest ago is evicted, and with it every cached block whose prefix runs
 *     through it.
 *   - A block is cached when it becomes full (at allocation for a prompt, when
 *     its last slot is reserved during decode) if the prefix before it is
 *     cached (or it is the first block) and its own prefix is not cached yet.
 *   - Prompt tokens found in the cache get slot -1 (pa_reshape_and_cache skips
 *     them); the others get block * block_size + offset.
 *   - Appending to a sequence whose last block is partly filled and referenced
 *     by other tables first moves it to a fresh copy: one (shared, fresh) pair
 *     is returned for pa_copy_blocks, to run before the new tokens are written.
 *   - Every call is all-or-nothing: PA_ERR_NO_BLOCKS and PA_ERR_ARG leave the
 *     manager unchanged.
 *
 * Conventions: all pointers are HOST pointers owned by the caller; sequence ids
 * are caller-chosen int64 values.  A manager is not thread-safe: one thread at
 * a time.  Status codes are those of pa.h plus PA_ERR_NO_BLOCKS.
 */
#ifndef PA_KV_MANAGER_H_
#define PA_KV_MANAGER_H_

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

#define PA_ERR_NO_BLOCKS 6 /* the pool has too few free blocks for the call */

typedef struct pa_kvm pa_kvm; /* opaque manager */

/*
 * pa_kvm_create -- a manager of `num_blocks` device blocks of `block_size`
 * slots and `num_host_blocks` (>= 0) blocks of host swap space.
 * prefix_caching != 0 turns on prefix caching (token ids are then required by
 * add/append).  Returns NULL on bad sizes or when out of host memory.
 */
PA_API pa_kvm* pa_kvm_create(int32_t num_blocks, int32_t block_size, int32_t prefix_caching,
                             int32_t num_host_blocks);

/* pa_kvm_destroy -- release the manager (NULL is allowed). */
PA_API void pa_kvm_destroy(pa_kvm* m);

/* Blocks an allocation can take now: free ones plus unreferenced cached ones. */
PA_API int32_t pa_kvm_num_free_blocks(const pa_kvm* m);

/*
 * pa_kvm_add_sequence -- a new sequence `seq_id` holding the prompt `tokens`
 * (n >= 0 token ids; may be NULL when prefix caching is off).
 *   slots          int64 [n], out: each prompt token's slot, -1 for tokens
 *                  whose block came from the prefix cache.
 *   cached_tokens  out (may be NULL): prompt tokens found in the cache (a
 *                  multiple of block_size).
 * PA_ERR_ARG: duplicate id, n < 0, NULL slots (n > 0) or NULL tokens with
 * prefix caching on.
 */
PA_API int pa_kvm_add_sequence(pa_kvm* m, int64_t seq_id, const int32_t* tokens, int32_t n,
                               int64_t* slots, int32_t* cached_tokens);

/*
 * pa_kvm_append_tokens -- reserve the slots of n >= 0 new tokens at the end of
 * a sequence (n = 1 for a decode step, a chunk for chunked prefill).
 *   tokens      int32 [n] token ids (may be NULL when prefix caching is off).
 *   slots       int64 [n], out.
 *   copy_pair   int64 [2], out: (src, dst) when the shared last block was moved
 *               to a fresh copy; *num_pairs (0 or 1) says whether it was.
 */
PA_API int pa_kvm_append_tokens(pa_kvm* m, int64_t seq_id, const int32_t* tokens, int32_t n,
                                int64_t* slots, int64_t* copy_pair, int32_t* num_pairs);

/*
 * pa_kvm_decode_step -- one new token for each of num_seqs sequences, in order
 * (the same as pa_kvm_append_tokens with n = 1 for each), all or nothing for
 * the whole batch.
 *   tokens      int32 [num_seqs] (may be NULL when prefix caching is off).
 *   slots       int64 [num_seqs], out: pa_reshape_and_cache's slot_mapping.
 *   copy_pairs  int64 [num_seqs][2], out: the copies to run first, packed;
 *               *num_pairs of them.
 * PA_ERR_ARG also for a sequence listed twice.
 */
PA_API int pa_kvm_decode_step(pa_kvm* m, const int64_t* seq_ids, int32_t num_seqs,
                              const int32_t* tokens, int64_t* slots, int64_t* copy_pairs,
                              int32_t* num_pairs);

/* pa_kvm_fork -- new sequence `child` sharing every block of `parent`. */
PA_API int pa_kvm_fork(pa_kvm* m, int64_t parent, int64_t child);

/*
 * pa_kvm_share_prefix -- new sequence `dst` holding the first n_blocks blocks of
 * `src` (0 <= n_blocks <= blocks of src); its length is
 * min(length of src, n_blocks * block_size).
 */
PA_API int pa_kvm_share_prefix(pa_kvm* m, int64_t src, int64_t dst, int32_t n_blocks);

/*
 * pa_kvm_share_blocks -- for each logical index idx[i] (a full block of `src`,
 * inside `dst`'s table), `dst`'s block there becomes `src`'s; the block `dst`
 * held loses a reference.  The indices are checked before anything changes.
 */
PA_API int pa_kvm_share_blocks(pa_kvm* m, int64_t src, int64_t dst, const int32_t* idx, int32_t n);

/* pa_kvm_free_sequence -- drop a finished sequence; its blocks lose a reference
 * (last block first). */
PA_API int pa_kvm_free_sequence(pa_kvm* m, int64_t seq_id);

/* Context length and number of blocks of a sequence (either pointer may be NULL). */
PA_API int pa_kvm_sequence_info(const pa_kvm* m, int64_t seq_id, int32_t* context_len,
                                int32_t* num_blocks);

/* The block table of a sequence into table[capacity]; PA_ERR_SHAPE if it does not fit. */
PA_API int pa_kvm_block_table(const pa_kvm* m, int64_t seq_id, int32_t* table, int32_t capacity);

/*
 * pa_kvm_batch -- the decode inputs of a batch: block_tables int32
 * [num_seqs][max_blocks] (entries past a sequence's blocks set to -1, never
 * read by the kernels) and context_lens int32 [num_seqs].  PA_ERR_SHAPE if a
 * table is longer than max_blocks.
 */
PA_API int pa_kvm_batch(const pa_kvm* m, const int64_t* seq_ids, int32_t num_seqs,
                        int32_t max_blocks, int32_t* block_tables, int32_t* context_lens);

/*
 * pa_kvm_batch_update -- the same for arrays that already hold this batch's
 * tables as they were before the last pa_kvm_decode_step of these sequences
 * (same order): a decode step changes only a sequence's last table entry (a
 * new block, or its copy), so only that entry and the length are written.
 */
PA_API int pa_kvm_batch_update(const pa_kvm* m, const int64_t* seq_ids, int32_t num_seqs,
                               int32_t max_blocks, int32_t* block_tables, int32_t* context_lens);

/*
 * pa_kvm_swap_out -- move a sequence that holds every one of its blocks alone
 * ("当大模型推理遇上内存瓶颈" 5.1 CPU swap space, 7.3 cold blocks to slower
 * storage): each block gets the lowest free host block, in table order; the
 * device blocks are released (last first; cached ones stay in the prefix cache)
 * and the table now lists host blocks.  pairs (int64 [capacity][2]) receives
 * the (device, host) pairs for pa_swap_blocks(PA_SWAP_OUT), run before the
 * device blocks are reused.  PA_ERR_ARG for a shared block or a swapped-out
 * sequence, PA_ERR_SHAPE if capacity is too small, PA_ERR_NO_BLOCKS if the
 * host space is short.  A swapped-out sequence can only be swapped in, freed or
 * inspected.
 */
PA_API int pa_kvm_swap_out(pa_kvm* m, int64_t seq_id, int64_t* pairs, int32_t capacity,
                           int32_t* num_pairs);

/*
 * pa_kvm_swap_in -- bring a swapped-out sequence back into fresh device blocks
 * (nothing is registered in the prefix cache); pairs receives the (host,
 * device) pairs for pa_swap_blocks(PA_SWAP_IN), run before the sequence is used.
 */
PA_API int pa_kvm_swap_in(pa_kvm* m, int64_t seq_id, int64_t* pairs, int32_t capacity,
                          int32_t* num_pairs);

/* Free blocks of host swap space. */
PA_API int32_t pa_kvm_num_free_host_blocks(const pa_kvm* m);

/* Tables referencing `block`, or -1 when it is out of range. */
PA_API int32_t pa_kvm_ref_count(const pa_kvm* m, int32_t block);

#ifdef __cplusplus
}
#endif

#endif /* PA_KV_MANAGER_H_ */
