/*
 * pa_pool.h -- host-side KV block pool: free list, reference counts,
 * per-sequence block tables, slot mappings and copy-on-write bookkeeping.
 *
 * This is the allocator that generates the layouts the device calls in pa.h
 * consume (block tables, slot mappings, copy pairs).  It runs on the host and
 * touches no GPU memory.  The behaviour follows
 *   "PagedAttention: fragmentation, blocks, block tables"
 *     section 1 "The block pool"    -- allocation pops the head of the free
 *        queue; a request that needs more blocks than are free is refused;
 *        freed blocks whose count reaches zero are put back at the FRONT of
 *        the queue, as one run keeping their release order; a released
 *        sequence gives its blocks back last block first;
 *     section 2 "The block table"   -- a sequence's table only grows at its
 *        tail; token p is found through entry p / B, at offset p % B;
 *     section 3 "The slot mapping"  -- slot = table[p / B] * B + p % B;
 *     the copy-on-write passage     -- a redirected tail block and its source
 *        both stay retained until the copy has been handed to the device;
 *     "Two kinds of references"     -- such a retention (a "pin") is kept
 *        apart from owner references (tables naming the block): the
 *        copy-on-write trigger counts owners only, and a block is free only
 *        when it has neither owners nor pins;
 *     "What should every allocator mutation preserve?" -- pa_pool_check;
 *   "Memory management", Code       -- append with copy-on-write: copy iff the
 *        tail is partial and shared; the copy's block counts against the
 *        free blocks; a refused append changes nothing.
 *
 * Ownership: the pool owns all of its state; every output array is caller
 * allocated.  Calls are not thread-safe on one pool; separate pools are
 * independent.  Every call that can fail returns a pa_pool status (0 = ok,
 * negative = error) and leaves the pool unchanged on failure.
 */
#ifndef PA_POOL_H
#define PA_POOL_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_pool pa_pool_t;

enum {
    PA_POOL_OK = 0,
    PA_POOL_EINVAL = -1,     /* bad argument (null pointer, negative count, id out of range) */
    PA_POOL_ENOSPACE = -2,   /* not enough free blocks; nothing changed */
    PA_POOL_ENOSEQ = -3,     /* unknown sequence id */
    PA_POOL_EEXIST = -4,     /* sequence id already in use */
    PA_POOL_EINVARIANT = -5, /* pa_pool_check found a broken invariant */
    PA_POOL_ERANGE = -6      /* output too small (table wider than width, capacity) */
};

/* Copy-on-write trigger.
 * PA_COW_SHARED    (default): copy iff the tail block is partially filled and
 *                  more than one table names it ("Memory management", Code).
 * PA_COW_INHERITED: copy iff the tail block is partially filled and this
 *                  sequence did not allocate it itself, i.e. on every partial
 *                  hit ("PagedAttention: fragmentation, blocks, block tables",
 *                  copy-on-write passage: the trigger is len % B != 0). */
enum { PA_COW_SHARED = 0, PA_COW_INHERITED = 1 };

/* A pool of num_blocks blocks of block_size tokens.  free_order, if not NULL,
 * is a permutation of 0..num_blocks-1 giving the initial free queue, head
 * first (NULL = ascending).  Returns NULL on a bad argument or a free_order
 * that is not a permutation. */
pa_pool_t *pa_pool_create(int64_t num_blocks, int32_t block_size, const int32_t *free_order,
                          int32_t cow_rule);
void pa_pool_destroy(pa_pool_t *pool);

/* New empty sequence. */
int pa_pool_seq_create(pa_pool_t *pool, int64_t seq_id);
/* Extend a sequence by n_tokens >= 0 tokens: allocates
 * ceil((len + n) / B) - num_blocks(seq) new blocks, plus one for a
 * copy-on-write redirect of a shared partial tail (queued as a (src, dst)
 * pair).  PA_POOL_ENOSPACE leaves everything unchanged. */
int pa_pool_append(pa_pool_t *pool, int64_t seq_id, int64_t n_tokens);
/* One scheduler step: pa_pool_append(seq_ids[i], n_tokens) for every listed
 * sequence, in order, as one call.  Either every append is done or, when the
 * free queue cannot hold them all (copy-on-write redirects included, each
 * decided with the earlier appends of the call applied), none is:
 * PA_POOL_ENOSPACE and nothing changed.  PA_POOL_EINVAL for a sequence listed
 * twice; PA_POOL_ENOSEQ for an unknown one (nothing changed). */
int pa_pool_append_batch(pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs, int64_t n_tokens);
/* The whole host side of a decode step in one call: pa_pool_append_batch,
 * then pa_pool_take_copies, pa_pool_step_slots, pa_pool_block_table_update
 * and pa_pool_seq_lens over the same sequences, with the same results.
 *   pairs_out   [pairs_capacity][2] int64: every queued copy pair (earlier
 *               ones first); *num_pairs receives their count.
 *   slots_out   [num_seqs * n_tokens] int64: the slots of each sequence's
 *               last n_tokens positions, in call order.
 *   table, synced, width, as pa_pool_block_table_update (pad already in place).
 *   lens_out    [num_seqs] int32 lengths after the step.
 * All or nothing: every check is made before anything changes.
 * PA_POOL_ENOSPACE (too few free blocks), PA_POOL_ENOSEQ, PA_POOL_EINVAL
 * (a sequence listed twice, or synced[r] past the sequence's blocks),
 * PA_POOL_ERANGE (pairs_capacity, width or an int32 length too small). */
int pa_pool_step(pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs, int64_t n_tokens, int64_t *pairs_out,
                 int64_t pairs_capacity, int64_t *num_pairs, int64_t *slots_out, int32_t width, int32_t *table,
                 int32_t *synced, int32_t *lens_out);
/* dst becomes a new sequence sharing every block of src (refcount + 1). */
int pa_pool_fork(pa_pool_t *pool, int64_t src, int64_t dst);
/* Drop the sequence; its blocks are freed in reverse order. */
int pa_pool_release(pa_pool_t *pool, int64_t seq_id);

/* Queued copy-on-write pairs. */
int64_t pa_pool_num_pending_copies(const pa_pool_t *pool);
/* Move all queued pairs into pairs_out ([n][2] int64, src then dst) and drop
 * the pin each endpoint held while queued.  Call it when the copies are
 * enqueued on the device, before the step's writes.  Returns the number of
 * pairs, or PA_POOL_ERANGE if capacity (in pairs) is too small. */
int64_t pa_pool_take_copies(pa_pool_t *pool, int64_t *pairs_out, int64_t capacity);

int64_t pa_pool_num_blocks(const pa_pool_t *pool);
int32_t pa_pool_block_size(const pa_pool_t *pool);
int64_t pa_pool_num_free(const pa_pool_t *pool);
/* Length in tokens / number of blocks of a sequence, or PA_POOL_ENOSEQ. */
int64_t pa_pool_seq_len(const pa_pool_t *pool, int64_t seq_id);
int64_t pa_pool_seq_num_blocks(const pa_pool_t *pool, int64_t seq_id);
/* Owner references (tables naming the block), or PA_POOL_EINVAL. */
int32_t pa_pool_refcount(const pa_pool_t *pool, int64_t block);
/* Pins (queued copies naming the block), or PA_POOL_EINVAL. */
int32_t pa_pool_pins(const pa_pool_t *pool, int64_t block);
/* Copy the free queue, head first, into out; returns its length or
 * PA_POOL_ERANGE. */
int64_t pa_pool_free_list(const pa_pool_t *pool, int32_t *out, int64_t capacity);

/* Rows of the device block table for num_seqs sequences: out is
 * [num_seqs][width] int32; entries past a sequence's block count are `pad`.
 * PA_POOL_ERANGE if a sequence holds more than width blocks. */
int pa_pool_block_table(const pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs,
                        int32_t width, int32_t pad, int32_t *out);
/* The same rows kept up to date in place, append-only ("PagedAttention:
 * fragmentation, blocks, block tables", section 2 "The block table": a
 * request's new block ids are appended to its row).  synced[r] is the number
 * of entries of row r written by earlier calls for the same sequence; a row
 * with synced[r] = 0 must hold `pad` everywhere (a fresh row, or one the
 * caller reset because it now names another sequence or a re-created id).  A
 * call writes only the old tail entry (a copy-on-write may have redirected
 * it) and the new entries, and sets synced[r] to the row's block count; the
 * rows then equal pa_pool_block_table's.  PA_POOL_ERANGE if a sequence holds
 * more than width blocks or synced[r] is outside [0, width]; PA_POOL_EINVAL
 * if synced[r] exceeds the sequence's block count (a sequence never loses
 * blocks, so the row was not reset); nothing is written on an error. */
int pa_pool_block_table_update(const pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs, int32_t width,
                               int32_t pad, int32_t *out, int32_t *synced);
/* int32 lengths of num_seqs sequences. */
int pa_pool_seq_lens(const pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs,
                     int32_t *out);
/* Slots of positions pos0 .. pos0+count-1 of one sequence (int64). */
int pa_pool_slots(const pa_pool_t *pool, int64_t seq_id, int64_t pos0, int64_t count,
                  int64_t *out);
/* The slot mapping of a step: for each sequence in order, the slots of its
 * last `tokens_per_seq` positions; out is [num_seqs * tokens_per_seq]. */
int pa_pool_step_slots(const pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs,
                       int64_t tokens_per_seq, int64_t *out);

/* Check the allocator invariants: the free queue and the referenced blocks
 * partition the pool; no block is on the free queue twice; every refcount
 * equals the number of table entries naming the block and every pin count
 * the number of queued-copy endpoints naming it; no table names a block
 * twice; every non-tail block is full and a tail holds 1..B tokens.
 * Returns PA_POOL_OK or PA_POOL_EINVARIANT. */
int pa_pool_check(const pa_pool_t *pool);

const char *pa_pool_status_str(int status);

#ifdef __cplusplus
}
#endif
#endif /* PA_POOL_H */
