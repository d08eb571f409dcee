/*
 * pagedkv.h -- C ABI of libpagedkv.so, the B200 (sm_100a) paged KV-cache
 * decode path.
 *
 * The method (PagedAttention) keeps each sequence's keys and values in
 * fixed-size physical blocks that may sit anywhere in a pool, and maps the
 * sequence's logical blocks to them through a per-sequence block table
 * ("PagedAttention Explained: Virtual Memory for the KV Cache", section "How
 * PagedAttention works", items 1-5).  This library provides the three device
 * operations of that design: the block-aware decode attention that gathers K
 * and V through the table (item 5), the append of new tokens' K/V into their
 * slots (section "The problem: the KV cache is big and unpredictable": the
 * cache grows by one entry per new token), and the block copy of
 * copy-on-write (section "Sharing blocks between sequences").
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pools: k_cache and v_cache are separate device arrays, each laid out
 *    [num_blocks][num_kv_heads][block_size][head_dim], row-major, elements of
 *    `dtype`.  One (block, kv head) slice is block_size*head_dim contiguous
 *    elements.  Both base pointers must be 16-byte aligned.
 *  - Token t of sequence s lives in physical block block_tables[s][t / bs] at
 *    slot t % bs; the physical slot index is block*bs + slot.
 *  - q and out are [num_seqs][num_heads][head_dim]; query head h reads kv head
 *    h / (num_heads / num_kv_heads) (contiguous groups, grouped-query
 *    attention; "Trade-offs and related techniques").
 *  - context_lens[s] counts every token the query attends, including tokens
 *    appended in this step; block_tables entries at index >=
 *    ceil(context_lens[s] / bs) are never read.
 *  - Attention is softmax(scale * q K^T) V over those tokens, accumulated in
 *    fp32, with out rounded to `dtype` (round to nearest even for bf16).  A
 *    sequence with context length 0 gets a zero output row.
 *  - All device pointers are owned by the caller; the library never frees
 *    them.  Every call is asynchronous on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream) and returns a status synchronously after
 *    host-side validation and the launch.  Nothing is thrown across the ABI.
 *  - Data-dependent faults found on the device (a table entry outside
 *    [0, num_blocks), a slot outside the pool, a context length outside
 *    [0, max_blocks_per_seq*bs], a wait that ran out of time) never trap: the
 *    kernel skips the affected work (a bad block is left out of the softmax, a
 *    bad sequence gets a zero row, a bad slot or pair is not written) and
 *    records the first such status in a per-device error word that
 *    pkv_get_device_error() returns.
 *
 * Supported shapes: head_dim in {64, 128}; block_size in {8, 16, 32};
 * num_heads / num_kv_heads in {1, 2, 4, 8}; dtype PKV_F32 or PKV_BF16.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum {
    PKV_OK = 0,
    PKV_ERR_NULL = -1,          /* a required pointer is NULL */
    PKV_ERR_INVALID = -2,       /* an argument is out of its documented range */
    PKV_ERR_UNSUPPORTED = -3,   /* a valid shape this build has no kernel for */
    PKV_ERR_CUDA = -4,          /* the CUDA runtime reported an error */
    PKV_ERR_WORKSPACE = -5,     /* decode workspace missing or too small */
    PKV_ERR_DEVICE_BOUNDS = -6, /* device word: a table entry, slot or length was out of range */
    PKV_ERR_TIMEOUT = -7,       /* device word: a bounded wait in a kernel ran out */
    PKV_ERR_OUT_OF_BLOCKS = -8  /* block manager: the free list cannot cover the request */
} pkv_status;

/* Element types of q, out, the pools and the new tokens.  PKV_FP8_E4M3
 * (OCP FP8 E4M3, one byte) is a cache type only: see the _fp8 calls. */
typedef enum { PKV_F32 = 0, PKV_BF16 = 1, PKV_FP8_E4M3 = 2 } pkv_dtype;

/* Kernels reported by the launch profiler. */
typedef enum {
    PKV_KERNEL_DECODE = 0, /* table walk, gather, QK^T, online softmax, PV, fused split-K merge */
    PKV_KERNEL_APPEND = 1,
    PKV_KERNEL_COPY_BLOCKS = 2,
    PKV_KERNEL_SWAP_BLOCKS = 3,
    PKV_KERNEL_KINDS = 4
} pkv_kernel_kind;

/*
 * Block-aware decode attention ("How PagedAttention works", item 5): for
 * every sequence s and query head h, out[s][h] = softmax(scale * q[s][h] .
 * K_s^T) V_s where K_s, V_s are the first context_lens[s] tokens of the
 * sequence gathered through block_tables (int32 [num_seqs][max_blocks_per_seq],
 * row-major).  This form takes bf16 data and partitions long contexts
 * automatically.
 *   - Pool bounds: its argument list carries no pool size, so table entries
 *     are checked only against 0.  An entry at or past the end of the pool
 *     is NOT detected: the kernel reads whatever device memory lies there,
 *     which can fault the context.  Use paged_attention_decode_ex, whose
 *     num_blocks turns such entries into device faults (block skipped, error
 *     word set).
 *   - Workspace: the library keeps one decode workspace per (device,
 *     stream), so calls on different streams never share one.  It is grown
 *     stream-ordered on the call's stream (cudaMallocAsync, zero fill, then
 *     cudaFreeAsync of the old buffer), which neither synchronises nor
 *     disturbs earlier launches on that stream.  A call made while the
 *     stream is being captured into a CUDA graph that would have to grow it
 *     returns PKV_ERR_WORKSPACE; inside capture, use paged_attention_decode_ex
 *     with a caller workspace.  The buffers live until the process exits.
 * Returns PKV_OK or a pkv_status.
 */
PKV_API int paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                           int num_heads, int num_kv_heads, int head_dim, int block_size,
                           int max_blocks_per_seq, float scale, void* stream);

/*
 * General form of paged_attention_decode.
 *   num_blocks        pool size; table entries outside [0, num_blocks) are
 *                     device faults (the block is skipped, error word set).
 *   dtype             pkv_dtype of q, out and the pools.
 *   partition_tokens  context tokens per CTA (split-K); a multiple of
 *                     block_size, at most 4096, or 0 for automatic (see
 *                     paged_attention_partition_tokens).  A sequence longer than one partition is split;
 *                     the last of its partitions to finish merges them all in
 *                     partition order, inside the same kernel.  Shorter ones
 *                     are written in one pass.
 *   workspace         device memory of at least
 *                     paged_attention_workspace_size(num_seqs, num_heads,
 *                     max_blocks_per_seq*block_size, head_dim, partition_tokens)
 *                     bytes, 256-byte aligned, owned by the caller.  It holds
 *                     at its start, in a region nothing else uses, the work
 *                     queue of the persistent fp8 kernel (64 bytes) and one
 *                     split-K merge counter per (sequence, kv head); then the
 *                     launch's schedule, then the partial results of split
 *                     sequences.
 *                     The schedule, where one is planned (see
 *                     pkv_set_longest_first), orders the grid's (sequence,
 *                     partition) units longest first; a one-CTA planning
 *                     kernel writes it and the decode kernel follows as a
 *                     programmatic dependent launch.  It changes which SM runs
 *                     a unit and when, never the arithmetic, so outputs are
 *                     the same bits with or without it.  Zero-fill the workspace (e.g.
 *                     cudaMemset) once before its first use.  Every call
 *                     leaves the queue and the counters it used at zero
 *                     again -- a call
 *                     whose kernel stopped on PKV_ERR_TIMEOUT too -- so the
 *                     same buffer serves later calls of any shape without
 *                     clearing.  (A batch of more than 65536 (sequence, kv
 *                     head) units also uses counters past that region; the
 *                     call clears those itself, on `stream`, before its
 *                     kernel.)  When no sequence is split, workspace may be
 *                     NULL: the grid then runs in index order, unplanned, one
 *                     CTA per (sequence, kv head, partition).  Two
 *                     calls in flight at once must not share a workspace.
 */
PKV_API int paged_attention_decode_ex(void* out, const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, const int32_t* context_lens,
                              int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, int max_blocks_per_seq, float scale, int num_blocks,
                              int dtype, int partition_tokens, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Partition size (tokens per CTA) paged_attention_decode_ex uses for these
 * arguments: partition_tokens itself, or the automatic choice when it is 0
 * (which depends on the kernel that serves the shape, and is at most 128
 * blocks where the persistent fp8 kernel serves it).  0 on bad sizes. */
PKV_API int paged_attention_partition_tokens(int num_seqs, int num_heads, int num_kv_heads,
                                             int head_dim, int block_size, int max_context,
                                             int dtype, int partition_tokens);

/*
 * Quantised KV cache ("What does PagedAttention change in LLM KV
 * allocation?", section "Sharing requires more than allocation": when the raw
 * KV data does not fit, cache quantization is one of the remedies).  The
 * pools hold fp8 e4m3 codes; one float scale per kv head (device arrays
 * k_scales, v_scales [num_kv_heads]) gives the stored value code * scale.  q
 * and out are bf16.  Otherwise exactly paged_attention_decode_ex (same
 * workspace, partitions, faults).  Tensor-core kernels serve it (both
 * products on e4m3 tensor cores over the codes as they land, q and the
 * probabilities each split into two e4m3 terms that keep 8 significant bits;
 * partitions a multiple of 128 tokens) with head_dim 128 and 1, 2, 4 or 8
 * query heads per kv head -- with a workspace and up to 4 heads in
 * persistent form (one CTA per SM slot taking units from the workspace's
 * queue, longest first; partitions of at most 128 blocks) -- and with
 * head_dim 64, 1, 2 or 4 query heads per kv head and an even number of kv
 * heads (one CTA per pair of kv heads).  Other shapes run on the CUDA-core
 * kernel, widening each code.  Every kernel reads half the bytes of a bf16
 * cache per token.
 */
PKV_API int paged_attention_decode_fp8(void* out, const void* q, const void* k_cache,
                                       const void* v_cache, const float* k_scales,
                                       const float* v_scales, const int32_t* block_tables,
                                       const int32_t* context_lens, int num_seqs, int num_heads,
                                       int num_kv_heads, int head_dim, int block_size,
                                       int max_blocks_per_seq, float scale, int num_blocks,
                                       int partition_tokens, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* Append to fp8 pools: new bf16 rows k, v [num_tokens][num_kv_heads][head_dim]
 * are stored as the e4m3 codes of x / scale (the division correctly rounded
 * in fp32; round to nearest even; magnitudes beyond 448 saturate to 448).
 * Slots as in kv_cache_append; head_dim a multiple of 16. */
PKV_API int kv_cache_append_fp8(void* k_cache, void* v_cache, const float* k_scales,
                                const float* v_scales, const void* k, const void* v,
                                const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                                int head_dim, int block_size, int num_blocks, void* stream);

/* Bytes of workspace paged_attention_decode_ex uses (the merge counters'
 * region, the schedule and, when sequences are split, the partial results);
 * 0 only for num_seqs <= 0.  With partition_tokens 0 the result covers any
 * automatic choice. */
PKV_API size_t paged_attention_workspace_size(int num_seqs, int num_heads, int max_context, int head_dim,
                                      int partition_tokens);

/*
 * Append new tokens ("The problem: the KV cache is big and unpredictable":
 * one new entry per token): for i < num_tokens with slot = slot_mapping[i]
 * >= 0, k_cache[slot / bs][g][slot % bs][:] = k[i][g][:] and likewise for v,
 * for every kv head g.  k and v are [num_tokens][num_kv_heads][head_dim];
 * slot_mapping is int64 [num_tokens]; -1 means "skip".  The copy is bit-exact.
 * Slots >= num_blocks*bs are device faults (not written).  Two tokens must not
 * name the same slot.  The append's kernel releases a kernel launched next
 * as a programmatic dependent at once (this library's decode kernels are
 * launched so, and wait for the append to finish before they read
 * anything); a caller's own kernel launched that way after it must likewise
 * wait (griddepcontrol.wait) before it reads the pools.
 */
PKV_API int kv_cache_append(void* k_cache, void* v_cache, const void* k, const void* v,
                    const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, int dtype, void* stream);

/*
 * Copy-on-write block copy ("Sharing blocks between sequences": the writer's
 * shared block is copied first, then its table is updated): for each pair i
 * of src_dst_pairs (int64 [num_pairs][2] = (src, dst)), the whole physical
 * block src -- every kv head and slot, keys and values -- is copied to dst.
 * Destinations must be distinct and no destination may also be a source (the
 * pairs are then independent and run in parallel).  Indices outside
 * [0, num_blocks) are device faults (pair skipped).  The caller updates its
 * block tables; the library never touches them.
 */
PKV_API int copy_blocks(void* k_cache, void* v_cache, const int64_t* src_dst_pairs, int num_pairs,
                int num_kv_heads, int head_dim, int block_size, int num_blocks, int dtype,
                void* stream);

/*
 * Decode attention for callers that cannot allocate device memory.  The pages
 * have no counterpart of this call: it is a property of this library, not of
 * the method.
 *
 * A serving engine usually gives its KV-block pool all the device memory left
 * after the weights, some host frameworks forbid allocations outside their own
 * allocator, and cudaMalloc / cudaFree may synchronise the device; such
 * callers cannot provide or let the library allocate the split-K workspace.
 * This call computes exactly what paged_attention_decode_ex computes (same
 * arguments without the workspace, same kernel, same results) and keeps the
 * split-K scratch in a fixed array of PKV_NOALLOC_SCRATCH_BYTES that is part
 * of the library's device image: every GPU that loads the library holds that
 * memory until the process exits.  It calls no allocating routine.
 *   - A batch whose scratch (paged_attention_workspace_size for the partition
 *     size chosen) exceeds PKV_NOALLOC_SCRATCH_BYTES returns
 *     PKV_ERR_WORKSPACE without launching anything; a larger partition_tokens
 *     lowers the need.
 *   - Each call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, which allocates nothing), so the address is
 *     right after a device reset too.  The first call on a device may load
 *     the library's device code there: make it before any stream capture.
 *   - All calls share the array and it keeps the last call's contents; each
 *     call clears the merge counters on its stream before its kernel.  Calls
 *     whose kernels overlap on the GPU (other streams, other threads) race on
 *     the array: order them.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
PKV_API int paged_attention_decode_noalloc(void* out, const void* q, const void* k_cache,
                                           const void* v_cache, const int32_t* block_tables,
                                           const int32_t* context_lens, int num_seqs,
                                           int num_heads, int num_kv_heads, int head_dim,
                                           int block_size, int max_blocks_per_seq, float scale,
                                           int num_blocks, int dtype, int partition_tokens,
                                           void* stream);

/*
 * Preemption by swapping ("Preemption and scheduling": move a sequence's
 * blocks to CPU memory and bring them back later): for each pair (src, dst)
 * of src_dst_pairs (int64 [num_pairs][2]), block src of the source pools
 * (src_k, src_v: [num_src_blocks][num_kv_heads][block_size][head_dim]) is
 * copied whole to block dst of the destination pools (same layout,
 * num_dst_blocks blocks).  Any pool and the pairs may be device memory or
 * page-locked (pinned) host memory; the copy is one kernel on `stream` that
 * reads or writes host pools over the host link through their device
 * mapping.  Pageable host memory is PKV_ERR_INVALID.  Bit-exact.  Indices
 * outside the pools are device faults (pair skipped).  Destinations must be
 * distinct and no destination may also be a source.
 */
PKV_API int swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                        const int64_t* src_dst_pairs, int num_pairs, int num_kv_heads,
                        int head_dim, int block_size, int num_src_blocks, int num_dst_blocks,
                        int dtype, void* stream);

/* Synchronise `stream`, then return in *code the current device's error word
 * (PKV_OK, PKV_ERR_DEVICE_BOUNDS or PKV_ERR_TIMEOUT) and clear it.  After
 * PKV_ERR_TIMEOUT the outputs of the decode launch that timed out are not
 * meaningful (they are finite: a stopped partition counts as empty), while
 * the pools, the workspaces and the context stay valid for later calls. */
PKV_API int pkv_get_device_error(void* stream, int* code);

/* Self-test of the failure path: launches one warp that waits, with the
 * kernels' bounded wait, on a barrier nothing arrives at; after timeout_us
 * microseconds (1 .. 1e6) the wait gives up and the device error word becomes
 * PKV_ERR_TIMEOUT (read it with pkv_get_device_error).  Nothing traps and the
 * context stays usable. */
PKV_API int pkv_selftest_bounded_wait(int timeout_us, void* stream);

/* Failure-path test hook: the limit, in microseconds, of the bounded waits
 * inside the decode kernels' pipelines (1 .. 1e6; 0 restores the default of
 * one second).  A limit far below a load's latency makes a real decode give
 * up, which is how the timeout path (PKV_ERR_TIMEOUT, a stopped CTA's turn on
 * its merge counter) is tested without a fault.  The wait that lets a
 * stopped CTA's own copies land keeps its one-second bound.  Process-wide;
 * read by each decode call at launch.  Returns the previous limit in
 * microseconds, or PKV_ERR_INVALID. */
PKV_API int pkv_set_wait_limit_us(int microseconds);

/* Debug builds.  libpagedkv_debug.so is this library compiled with
 * -DPKV_DEBUG: every index the kernels derive from the inputs (schedule
 * entries, units, copy sources and destinations, workspace and output rows)
 * is checked right before its use, and a failed check records
 * PKV_ERR_DEVICE_BOUNDS in the error word and its source line, then skips the
 * access instead of reading or writing out of bounds.  pkv_debug_build()
 * returns 1 in that build, 0 in the release one.  pkv_debug_failed_line()
 * synchronises `stream`, then returns in *line the source line of the first
 * failed check since the last read (0: none; always 0 in release builds) and
 * clears it. */
PKV_API int pkv_debug_build(void);
PKV_API int pkv_debug_failed_line(void* stream, int* line);

/* Static English text of a status code. */
PKV_API const char* pkv_status_string(int status);

/*
 * Launch profiler.  When enabled, every kernel launch is bracketed by CUDA
 * events recorded on its own stream.  pkv_profile_read() waits for the
 * recorded launches of `kind` and returns their count and summed device time
 * in milliseconds; pkv_profile_reset() forgets every record.
 */
PKV_API int pkv_profile_enable(int on);
PKV_API int pkv_profile_read(int kind, long long* launches, double* total_ms);
PKV_API int pkv_profile_reset(void);

/* Choose the decode kernel where a tensor-core one applies (partitions a
 * multiple of 128 tokens; head_dim 128 with bf16 caches and 2, 4 or 8 query
 * heads per kv head, or fp8 caches and 1, 2, 4 or 8; head_dim 64 with fp8
 * caches, 1, 2 or 4 and an even number of kv heads): 1 (default) runs the
 * tensor-core kernel (tcgen05 MMAs into tensor memory), 0 the CUDA-core
 * kernels that serve every other shape (bf16 caches with one query head per
 * kv head and head_dim 64 or 128 stream K and V through registers; the rest
 * stage them in shared memory).  All compute the same attention; returns the
 * previous setting.  Process-wide. */
PKV_API int pkv_set_tensor_core_gqa(int enable);

/* Schedule of the decode grid (calls with a workspace; see
 * paged_attention_decode_ex): 1 (default) plans longest first where that
 * pays -- the tensor-core kernels with 2 to 4 partitions per sequence, whose
 * index order would leave the partitions only long sequences have for the
 * end of the launch, the persistent fp8 kernel, whose queue then hands out
 * the shortest units last, and the head_dim-64 fp8 kernel -- and runs every
 * other launch in index order; 2 plans
 * every launch; 0 none.  All give the same bits; only the time differs.
 * Process-wide; returns the previous mode, or PKV_ERR_INVALID. */
PKV_API int pkv_set_longest_first(int mode);

/* Kernels launched by this library in this process so far (all kinds). */
PKV_API unsigned long long pkv_launch_count(void);

/* Library version, major*10000 + minor*100 + patch. */
PKV_API int pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
