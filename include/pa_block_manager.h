/*
 * Host block manager for the paged KV cache (part of libpa; host-only, no CUDA call).
 *
 * It owns the mapping the decode kernels read: for every sequence, the list of
 * physical blocks that hold its tokens in order (the page table: "Sequence -> [page
 * indices]", "IO-5 vLLM Paged Attention" note, section 3).  It follows the pages'
 * description of the block manager:
 *   - blocks are handed out on demand and returned as soon as a sequence ends
 *     ("PagedAttention" summary, features 1 and 4; "PagedAttention and dynamic memory
 *     management" blog, BlockSpaceManager: pool initialisation, "can this request be
 *     allocated?", blocks_needed = ceil(seq_len / block_size));
 *   - several sequences may share blocks (features 2: parallel sampling over one
 *     prompt) -- a block carries a reference count;
 *   - appending into a shared, partially filled block first gives the writer a
 *     private copy (copy-on-write), emitted as a (src, dst) pair for pa_copy_blocks;
 *   - block_usage_ratio = used blocks / pool blocks (the blog's deployment tip).
 *
 * The decode step that uses it:  pa_bm_append_slots (one new token per sequence)
 * -> pa_copy_blocks(pairs) -> pa_kv_write(slot_mapping) -> pa_decode(tables, lens);
 * or, with the copies done by the decode itself, pa_bm_append_slots_cow ->
 * pa_decode_cow(tables, lens, copy list, new tokens).  pa_bm_block_tables fills the
 * table and length arrays for the listed sequences.
 *
 * Not thread-safe: one manager per engine thread.  Operations other than swap-in and
 * free on a swapped-out sequence return PA_ERR_INVALID_ARG.  Sequence ids are caller-chosen
 * int64 values.  Errors: PA_ERR_INVALID_ARG (null pointer, unknown or duplicate
 * sequence id, bad size), PA_ERR_NO_FREE_BLOCK (the pool cannot satisfy the request),
 * PA_ERR_HOST_ALLOC (a host allocation for the manager's bookkeeping failed).  A call
 * that returns an error has changed nothing; no exception crosses this interface.
 */
#ifndef PA_BLOCK_MANAGER_H
#define PA_BLOCK_MANAGER_H

#include <stdint.h>

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

/* Pool of num_blocks blocks of block_size tokens; NULL on bad arguments or when the
 * host memory for the pool's bookkeeping cannot be allocated. */
pa_block_manager *pa_bm_create(int num_blocks, int block_size);
void pa_bm_destroy(pa_block_manager *bm);

/*
 * Sliding window (the blog's BlockSpaceManager(sliding_window=...)): with window W > 0
 * a sequence of length L only needs its last W positions, [max(0, L - W), L), so a
 * block that lies wholly before them ((j + 1) * bs <= L - W for table index j) is
 * returned to the pool at the sequence's next pa_bm_append_slots and its table entry
 * becomes -1; pa_decode with the same sliding_window never reads such an entry.  A
 * new sequence takes the blocks of all its tokens (its prompt is written and
 * attended in full, as pa_prefill with a window needs the W - 1 tokens before its
 * first query).  Blocks that fall out of the window during pa_bm_append_slots are
 * given back after the whole batch has its slots (so its all-or-nothing check counts
 * only blocks that were free before the call).  pa_bm_slot of a released position is
 * -1.
 * Only while the manager holds no sequence; 0 = whole contexts (the default).
 */
pa_status pa_bm_set_sliding_window(pa_block_manager *bm, int window);

/* ceil(num_tokens / block_size) (the blog's blocks_needed); -1 on bad arguments. */
int pa_bm_blocks_needed(int num_tokens, int block_size);

int pa_bm_num_free_blocks(const pa_block_manager *bm);

/* used blocks / pool blocks. */
double pa_bm_usage_ratio(const pa_block_manager *bm);

/* 1 if a new sequence of num_tokens tokens fits in the free blocks, else 0. */
int pa_bm_can_allocate(const pa_block_manager *bm, int num_tokens);

/* New sequence holding num_tokens tokens (a prompt): ceil(num_tokens / bs) fresh
 * blocks, reference count 1.  The caller writes those tokens with pa_kv_write at
 * slots pa_bm_slot(seq_id, 0 .. num_tokens-1). */
pa_status pa_bm_allocate(pa_block_manager *bm, int64_t seq_id, int num_tokens);

/* child := a sequence that shares all of parent's blocks and length (each block's
 * reference count + 1). */
pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent_id, int64_t child_id);

/* Ends a sequence: reference counts - 1; blocks that reach 0 return to the pool. */
pa_status pa_bm_free(pa_block_manager *bm, int64_t seq_id);

/*
 * Reserves the slot of one new token for each of the n listed sequences (distinct
 * ids), in order: a fresh block when the token starts a block; a private copy of the
 * last block when it is shared and partially filled (pair (old, new) appended to
 * copy_pairs, int64 [max_pairs][2]); otherwise the next free slot of the last block.
 * slot_mapping[i] receives the slot (block * bs + offset); *num_pairs the number of
 * pairs.  All or nothing: if the pool cannot cover the whole batch (or max_pairs is
 * too small) nothing changes and PA_ERR_NO_FREE_BLOCK / PA_ERR_INVALID_ARG returns.
 */
pa_status pa_bm_append_slots(pa_block_manager *bm, const int64_t *seq_ids, int n,
                             int64_t *slot_mapping, int64_t *copy_pairs, int max_pairs,
                             int *num_pairs);

/*
 * pa_bm_append_slots for a decode step that makes its copies itself (pa_decode_cow):
 * the same reservations, with each private copy reported per sequence instead of as a
 * pair.  cow, int32 [n][3], receives for sequence i (source block, logical index of
 * its last block, rows of that block filled before the new token) when its last block
 * was copied, else (-1, 0, 0) -- pa_decode_cow's copy list, in the order of seq_ids;
 * *num_copies the number of copies.  The new token goes to the row past the copied
 * ones, so the copy and the token's cache write touch different rows.  Errors and
 * all-or-nothing as pa_bm_append_slots.
 */
pa_status pa_bm_append_slots_cow(pa_block_manager *bm, const int64_t *seq_ids, int n,
                                 int64_t *slot_mapping, int32_t *cow, int *num_copies);

/* Slot of token position pos of a sequence (block * bs + offset), -1 if out of range. */
int64_t pa_bm_slot(const pa_block_manager *bm, int64_t seq_id, int pos);

/* Context length of a sequence, -1 if unknown. */
int pa_bm_seq_len(const pa_block_manager *bm, int64_t seq_id);

/* Reference count of a physical block (0 = free), -1 if out of range. */
int pa_bm_block_refcount(const pa_block_manager *bm, int block);

/*
 * Host pool for preemption (the blog's num_cpu_blocks; the summary's preemptive
 * scheduling): a preempted group of sequences is swapped out to host blocks and later
 * back in, with pa_swap_blocks moving the data.  A swapped-out sequence can only be
 * swapped in or freed.
 */
pa_status pa_bm_set_cpu_pool(pa_block_manager *bm, int num_cpu_blocks); /* once */
int pa_bm_num_free_cpu_blocks(const pa_block_manager *bm);

/* 1 if the sequence's blocks are in the host pool, 0 if on the GPU, -1 if unknown. */
int pa_bm_is_swapped(const pa_block_manager *bm, int64_t seq_id);

/*
 * Swap out the n listed GPU-resident sequences: every distinct GPU block they use gets
 * one host block (so blocks shared inside the group stay shared), pairs (gpu block,
 * host block) go to pairs [max_pairs][2] for pa_swap_blocks(host pool <- GPU cache),
 * and the GPU blocks return to the GPU pool.  The group must hold every reference to
 * its blocks (a block also used by an unlisted sequence: PA_ERR_INVALID_ARG).  All or
 * nothing (PA_ERR_NO_FREE_BLOCK when the host pool is short).
 */
pa_status pa_bm_swap_out(pa_block_manager *bm, const int64_t *seq_ids, int n, int64_t *pairs,
                         int max_pairs, int *num_pairs);

/* The reverse: host blocks -> fresh GPU blocks, pairs (host block, gpu block) for
 * pa_swap_blocks(GPU cache <- host pool).  All or nothing. */
pa_status pa_bm_swap_in(pa_block_manager *bm, const int64_t *seq_ids, int n, int64_t *pairs,
                        int max_pairs, int *num_pairs);

/* For the n listed sequences: block_tables [n][width] (unused entries -1) and
 * context_lens [n], host arrays ready to copy to the device for pa_decode.
 * PA_ERR_INVALID_ARG if a table does not fit in width. */
pa_status pa_bm_block_tables(const pa_block_manager *bm, const int64_t *seq_ids, int n,
                             int32_t *block_tables, int width, int32_t *context_lens);

#ifdef __cplusplus
}
#endif

#endif /* PA_BLOCK_MANAGER_H */
