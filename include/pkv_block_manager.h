/*
 * pkv_block_manager.h -- host-side block manager of libpagedkv.so.
 *
 * Keeps the bookkeeping the pages describe around the device kernels:
 *  - a pool of fixed-size physical blocks and a free list ("PagedAttention
 *    Explained: Virtual Memory for the KV Cache", section "How PagedAttention
 *    works", items 1 and 4: every block the same size, and a new physical
 *    block only when the sequence's last block fills -- nothing reserved in
 *    advance);
 *  - one block table per sequence (items 2 and 3);
 *  - reference counts, forking and copy-on-write (section "Sharing blocks
 *    between sequences": sampled completions and beams share blocks; a
 *    writer whose block is shared gets a copy first and its table is
 *    updated);
 *  - release when a request finishes ("What does PagedAttention change in
 *    LLM KV allocation?", section "Calculate unused block space");
 *  - swapping a sequence's blocks to a host pool and back, and the choice of
 *    the most recently arrived sequence as the victim (section "Preemption
 *    and scheduling");
 *  - the counters that page says to measure: allocated blocks, used token
 *    positions, preemptions, live sequences.
 * The manager only decides; the copies it asks for run on the device with
 * copy_blocks (copy-on-write) and swap_blocks (swapping), declared in
 * pagedkv.h.  It is not thread-safe: use one host thread per manager.
 */
#ifndef PKV_BLOCK_MANAGER_H
#define PKV_BLOCK_MANAGER_H

#include <stdint.h>

#include "pagedkv.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pkv_block_manager pkv_block_manager;

/* Counters of one manager.  "Physical" counts each block once however many
 * sequences share it; "logical" sums over sequences. */
typedef struct {
    int64_t num_blocks;          /* device pool size */
    int64_t free_blocks;         /* device blocks on the free list */
    int64_t used_blocks;         /* device blocks referenced by at least one sequence */
    int64_t allocated_slots;     /* used_blocks * block_size */
    int64_t used_slots;          /* device slots holding a token of at least one sequence */
    int64_t logical_allocated;   /* sum over live sequences of blocks * block_size */
    int64_t logical_used;        /* sum over live sequences of their lengths */
    int64_t live_sequences;      /* sequences resident on the device */
    int64_t swapped_sequences;   /* sequences whose blocks are in the host pool */
    int64_t host_free_blocks;    /* host pool blocks on its free list */
    int64_t preemptions;         /* swap-outs so far */
    int64_t copy_on_write;       /* copy-on-write pairs handed out so far */
} pkv_bm_stats;

/* Create a manager for a device pool of num_blocks blocks of block_size tokens
 * and a host pool of num_host_blocks blocks (0: no swapping).  free_order, if
 * not NULL, is a permutation of [0, num_blocks) giving the order in which
 * free device blocks are handed out (NULL: ascending).  Blocks released later
 * are reused first.  Returns NULL on bad arguments. */
PKV_API pkv_block_manager* pkv_bm_create(int num_blocks, int block_size, int num_host_blocks,
                                         const int32_t* free_order);
PKV_API void pkv_bm_destroy(pkv_block_manager* bm);

/* A new, empty sequence; returns its id (>= 0) or a negative status. */
PKV_API int pkv_bm_add_sequence(pkv_block_manager* bm);

/* A new sequence sharing every block of `parent` (each refcount + 1) and its
 * length (parallel sampling, beam forks).  Returns the id or a status. */
PKV_API int pkv_bm_fork(pkv_block_manager* bm, int parent);

/*
 * Make room for n new tokens at the end of `seq`: their physical slots
 * (block * block_size + offset) go to slots[0..n).  If the first new token
 * lands in the sequence's last block and that block is shared (refcount >
 * 1), the block is copied first: a fresh block replaces it in this sequence's
 * table, the old block's refcount drops, and the pair (old, new) is written
 * to cow_pairs (int64 [max_pairs][2]); *n_pairs counts the pairs (0 or 1).
 * New blocks are taken from the free list only when the last one is full.
 * PKV_ERR_OUT_OF_BLOCKS when the free list cannot cover the request (nothing
 * changes: preempt and retry).  The caller runs copy_blocks on the pairs,
 * then kv_cache_append on the slots, then decodes with the exported tables.
 */
PKV_API int pkv_bm_append(pkv_block_manager* bm, int seq, int n, int64_t* slots,
                          int64_t* cow_pairs, int max_pairs, int* n_pairs);

/* The request finished: drop the sequence; its blocks' refcounts drop and
 * blocks no longer referenced return to the free list. */
PKV_API int pkv_bm_free(pkv_block_manager* bm, int seq);

/* Block tables (int32 [n][max_blocks], -1 past the sequence's blocks) and
 * context lengths of the listed live sequences.  PKV_ERR_INVALID if a table
 * does not fit max_blocks or a sequence is not resident. */
PKV_API int pkv_bm_tables(const pkv_block_manager* bm, const int32_t* seqs, int n,
                          int max_blocks, int32_t* tables, int32_t* context_lens);

/* Length (tokens) of a sequence, or a negative status. */
PKV_API int pkv_bm_length(const pkv_block_manager* bm, int seq);

/* The live sequence that arrived last (the preemption victim), or -1. */
PKV_API int pkv_bm_pick_victim(const pkv_block_manager* bm);

/*
 * Preempt `seq` by swapping: each of its device blocks gets a host-pool
 * block; the (device_block, host_block) pairs go to pairs (int64
 * [max_pairs][2], *n_pairs of them) for swap_blocks(device -> host); then the
 * device blocks are released as by pkv_bm_free, and the sequence keeps its
 * length and host table.  PKV_ERR_OUT_OF_BLOCKS if the host pool is too small.
 */
PKV_API int pkv_bm_swap_out(pkv_block_manager* bm, int seq, int64_t* pairs, int max_pairs,
                            int* n_pairs);

/* Bring a swapped sequence back: fresh device blocks for each host block;
 * (host_block, device_block) pairs for swap_blocks(host -> device); the host
 * blocks return to the host free list.  PKV_ERR_OUT_OF_BLOCKS if the device
 * pool is too small (nothing changes). */
PKV_API int pkv_bm_swap_in(pkv_block_manager* bm, int seq, int64_t* pairs, int max_pairs,
                           int* n_pairs);

PKV_API int pkv_bm_get_stats(const pkv_block_manager* bm, pkv_bm_stats* out);

#ifdef __cplusplus
}
#endif

#endif /* PKV_BLOCK_MANAGER_H */
