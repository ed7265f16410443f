/*
 * pa.h -- C ABI of the B200 paged-KV-cache attention library (libpa.so).
 *
 * The library implements the data-parallel hot path of PagedAttention decode:
 * the KV cache is stored in fixed-size blocks scattered over a physical pool,
 * each sequence owns a block table mapping its logical blocks to physical
 * ones, and attention for the newly generated token reads K/V through that
 * table; around it, the cache write, copy-on-write block copies, a host block
 * manager (with prefix caching across requests) and chunked-prefill attention
 * over the same pool.  Sources (cited by page title and section):
 *
 *   [P1] "Why OS Virtual Memory Paging Saved LLM Inference: The vLLM
 *        Breakthrough" -- section 2 "The PagedAttention Architecture" (KV
 *        blocks, block table, on-demand allocation, the kernel that looks up
 *        physical blocks and fetches K/V on the fly) and section 3
 *        "Copy-on-Write for Prompt Sharing".
 *   [P3] "Can OS paging techniques reduce LLM serving memory waste?" --
 *        second paragraph (block-by-block attention over non-contiguous
 *        blocks; a KV cache manager with one block table per request;
 *        sharing of blocks within and across a batch).
 *
 * Conventions for every call below
 *   - Device pointers are owned by the caller (e.g. torch tensors); the
 *     library never allocates, frees or keeps device memory (the one fixed
 *     array of pa_paged_decode_attention_no_alloc is part of the loaded
 *     module).  Host pointers are read or written only during the call.
 *   - Tensors are dense, row-major ("C-contiguous") in the layouts given.
 *   - Pool layout: k_cache / v_cache are [num_blocks, num_kv_heads,
 *     block_size, head_dim] elements of `dtype`; token t of a sequence lives
 *     in block block_tables[s][t / block_size] at offset t % block_size.
 *     A "slot" is block * block_size + offset.
 *   - Kernels are launched asynchronously on `stream` (NULL = the legacy
 *     default stream) and the call returns without synchronising.  Device
 *     pointers must be 16-byte aligned.
 *   - Return value: PA_OK (0) or a negative pa_status.  Argument errors are
 *     detected on the host before anything is launched.  Bad indices found
 *     on the device (a block id outside the pool, a slot outside the pool, a
 *     context length beyond the table) never fault: the access is skipped and
 *     a bit is set in a sticky device error word read by pa_device_error().
 *   - Supported shapes: head_dim in {64, 128}; block_size in {16, 32};
 *     num_q_heads a multiple of num_kv_heads with group size
 *     num_q_heads / num_kv_heads <= 16; query head h reads kv head
 *     h / (num_q_heads / num_kv_heads).  Others return PA_ERR_UNSUPPORTED.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st *pa_stream_t;

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_ARG = -1,           /* invalid argument (null pointer, negative size, ...) */
  PA_ERR_UNSUPPORTED = -2,   /* valid but not implemented shape */
  PA_ERR_NO_BLOCKS = -3,     /* block manager: free list too short */
  PA_ERR_SEQ = -4,           /* block manager: unknown or duplicate sequence id */
  PA_ERR_CUDA = -5,          /* a CUDA runtime call failed */
  PA_ERR_DEVICE_BOUNDS = -6, /* pa_device_error(): a device-side check fired */
  PA_ERR_WORKSPACE = -7      /* workspace too small or misaligned */
} pa_status;

/* Bits of the sticky device error word. */
#define PA_DEVERR_BLOCK_ID 0x1u    /* block table entry outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT_LEN 0x2u /* context_len < 0 or > max_blocks_per_seq * block_size */
#define PA_DEVERR_SLOT 0x4u        /* slot_mapping entry >= num_blocks * block_size */
#define PA_DEVERR_COPY_PAIR 0x8u   /* copy_blocks pair outside [0, num_blocks) */
#define PA_DEVERR_TIMEOUT 0x10u    /* a bounded wait on an asynchronous copy gave up */
#define PA_DEVERR_RANGE 0x20u      /* prefill over a bf16 cache: an output row came out not
                                      finite -- a V value beyond fp16's range (|v| >= 65520)
                                      or a non-finite q, K or V element */

/* Human-readable name of a pa_status value (static string). */
const char *pa_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int pa_version(void);

/*
 * Write each step's new K/V into the slots its block table assigns
 * ([P1] section 2, on-demand allocation: blocks are taken one by one as new
 * tokens arrive, and each token's K/V goes into its slot).
 *
 *   key, value     [num_tokens, num_kv_heads, head_dim] of dtype (device)
 *   k_cache,v_cache pool [num_blocks, num_kv_heads, block_size, head_dim] (device)
 *   slot_mapping   int64 [num_tokens] (device); token t goes to
 *                  cache[slot / block_size, :, slot % block_size, :];
 *                  slot < 0 skips the token; slot >= num_blocks * block_size
 *                  is skipped and sets PA_DEVERR_SLOT.
 * Two tokens with the same slot in one call: which one lands is undefined.
 * num_tokens == 0 launches nothing.
 */
int pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                         const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                         pa_stream_t stream);

/*
 * Bytes of device workspace that cover every pa_paged_decode_attention or
 * pa_decode_step launch on the current device for these sizes, whatever
 * pa_decode_tuning selects (0 on error): an upper bound, sized for the
 * largest grid (4 CTAs per SM); the default launch needs less.  The
 * workspace holds the per-warp split-context partial results and their
 * descriptors; its contents need no initialisation and are dead after the
 * call.
 */
size_t pa_paged_decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads,
                                       int head_dim, int block_size, int max_context_len);

/*
 * PagedAttention decode ([P1] section 2: for a newly generated token the
 * kernel looks up the physical blocks in the block table and fetches K/V
 * from non-contiguous memory; [P3] second paragraph: attention computed
 * block by block).  For every sequence s and query head h, with
 * kh = h / (num_q_heads / num_kv_heads) and L = context_lens[s]:
 *
 *   out[s, h, :] = sum_t softmax_t(scale * <q[s, h, :], K_s[t]>) V_s[t],
 *   K_s[t] = k_cache[block_tables[s][t / B], kh, t % B, :], t = 0 .. L-1,
 *
 * accumulated in fp32.  L counts every cached token of the sequence, the one
 * written this step included; L == 0 gives a zero row.  Long sequences are
 * split across warps (split context) and the partial softmax states are
 * merged by a second kernel launched on the same stream.  If a bounded wait
 * of the call runs out (PA_DEVERR_TIMEOUT, see pa_set_wait_limit), its output
 * rows are undefined.
 *
 *   out           fp32 [num_seqs, num_q_heads, head_dim] (device, written)
 *   q             dtype [num_seqs, num_q_heads, head_dim] (device)
 *   k_cache,v_cache pool as above, dtype (device)
 *   block_tables  int32 [num_seqs, max_blocks_per_seq] (device); entries at
 *                 index >= ceil(L / B) are never read
 *   context_lens  int32 [num_seqs] (device)
 *   max_context_len an upper bound on context_lens (host value, used for
 *                 sizing only)
 *   workspace     device scratch of at least pa_paged_decode_workspace_bytes()
 *                 bytes, 256-byte aligned; must not be shared by calls that
 *                 may run concurrently.
 */
int pa_paged_decode_attention(float *out, const void *q, const void *k_cache,
                              const void *v_cache, const int32_t *block_tables,
                              const int32_t *context_lens, float scale, int num_kv_heads,
                              int num_seqs, int num_q_heads, int head_dim, int block_size,
                              int max_blocks_per_seq, int max_context_len, int num_blocks,
                              pa_dtype dtype, void *workspace, size_t workspace_bytes,
                              pa_stream_t stream);

/*
 * One decode step fused into one launch: the cache write of every sequence's
 * newest token (as pa_reshape_and_cache would do it) and the decode attention
 * over all of its tokens (as pa_paged_decode_attention).  Follows the same
 * pages: [P1] section 2 (on-demand allocation of the new token's slot; the
 * kernel that reads K/V through the block table for the new token).
 *
 *   k_new, v_new  dtype [num_seqs, num_kv_heads, head_dim] (device): the K/V
 *                 of token L-1 of each sequence (L = context_lens[s]); it is
 *                 stored at position L-1 of the sequence's block table, i.e.
 *                 in block block_tables[s][(L-1) / B] at offset (L-1) % B,
 *                 and attention uses it directly.  Sequences with L == 0 have
 *                 no new token and get a zero row.
 *   k_cache, v_cache are written (that one slot per sequence and kv head).
 * All other arguments as for pa_paged_decode_attention.  The result equals
 * pa_reshape_and_cache with slot_mapping[s] = that position, followed by
 * pa_paged_decode_attention; the block holding position L-1 must be the
 * sequence's own (not shared: copy it with pa_copy_blocks first).
 */
int pa_decode_step(float *out, const void *q, const void *k_new, const void *v_new,
                   void *k_cache, void *v_cache, const int32_t *block_tables,
                   const int32_t *context_lens, float scale, int num_kv_heads, int num_seqs,
                   int num_q_heads, int head_dim, int block_size, int max_blocks_per_seq,
                   int max_context_len, int num_blocks, pa_dtype dtype, void *workspace,
                   size_t workspace_bytes, pa_stream_t stream);

/*
 * Allocation-free variant of pa_paged_decode_attention (no counterpart in the
 * pages: an integration convenience).  Same arguments, same result, but no
 * workspace argument: the split-context scratch lives in a fixed array of
 * PA_NO_ALLOC_SCRATCH_BYTES compiled into the library, which every GPU that
 * loads the library keeps until the process exits.  It is meant for callers
 * that cannot allocate device memory themselves -- a plugin that only gets
 * input and output buffers from a host framework owning all device memory,
 * or a latency-critical caller where cudaMalloc (which may synchronise the
 * device, or fail under memory pressure) is not allowed.  The call itself
 * makes no device allocation and frees nothing.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call on a device shares the one array, which keeps the
 * last call's contents: every partial result the call reads back is written
 * by the same call first, so nothing needs clearing between calls (after a
 * call whose wait ran out, PA_DEVERR_TIMEOUT, the output is undefined
 * anyway).  Calls that may overlap on the GPU -- on different streams, or
 * from different threads -- race on the array and must be serialised by the
 * caller.  Returns PA_ERR_WORKSPACE, launching nothing, when the launch
 * would need more than PA_NO_ALLOC_SCRATCH_BYTES; otherwise as
 * pa_paged_decode_attention.
 *
 * What fits: the scratch of a launch is about 8 * W * (G * (head_dim + 2) + 8)
 * bytes for W warps in the grid and G = num_q_heads / num_kv_heads (it does
 * not depend on the number of sequences or their lengths).  With the default
 * launch shape on a 148-SM B200 (W = 1184 for G >= 2 at block_size 16 or at
 * head_dim 64, W = 592 at head_dim 128 with block_size 32, W = 1776 for
 * G = 1) every supported shape fits except head_dim 128, block_size 16 with
 * G = 14, 15 or 16.  pa_paged_decode_workspace_bytes is an upper bound over
 * all tunings, not this launch's need: it exceeds the array from G = 7 at
 * head_dim 128 although those calls succeed.
 */
#define PA_NO_ALLOC_SCRATCH_BYTES (16u << 20)
int pa_paged_decode_attention_no_alloc(float *out, const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       const int32_t *context_lens, float scale,
                                       int num_kv_heads, int num_seqs, int num_q_heads,
                                       int head_dim, int block_size, int max_blocks_per_seq,
                                       int max_context_len, int num_blocks, pa_dtype dtype,
                                       pa_stream_t stream);

/*
 * Override the decode launch heuristics for this process (0 = automatic):
 * stages of the per-warp copy ring, CTAs per SM, and the fewest tiles
 * ((sequence, kv head, block) units) a warp is given.  Affects calls made
 * after it; results stay within the attention tolerance but the split points,
 * hence the rounding, change.  No counterpart on the pages: a tuning knob.
 */
int pa_decode_tuning(int nstage, int ctas_per_sm, int min_tiles_per_warp);

/*
 * Limit, in nanoseconds of wall time, of every bounded wait inside the
 * kernels launched after this call (decode, decode step, prefill): a wait on
 * an asynchronous copy or on the tensor cores that lasts longer gives up,
 * sets PA_DEVERR_TIMEOUT, lets the copies and MMAs already issued complete
 * (those drains keep their own fixed bounds, so nothing lands after a CTA
 * has left) and returns; the output rows of that call are then undefined.
 * ns == 0 restores the default of 2 s, far above any copy's latency; a tiny
 * limit makes the waits run out on purpose, which is how failure detection
 * is tested without faulting or hanging the GPU.  Limits under 1 ms are
 * polled (no sleeping wait) and counted in SM clock cycles at 2 per ns, so
 * they run out no earlier than asked at clocks up to 2 GHz.  Process-wide;
 * returns PA_ERR_ARG for ns < 0.  No counterpart on the pages.
 */
int pa_set_wait_limit(long long ns);

/*
 * Copy-on-write block copies ([P1] section 3: a branch that writes into a
 * shared block gets its own private block, which starts as a copy).
 *
 *   block_mapping int64 [num_pairs, 2] (device): (src, dst) physical block
 *                 ids; cache[dst] = cache[src] for every kv head, in both the
 *                 K and the V pool.  A pair with an id outside [0, num_blocks)
 *                 is skipped and sets PA_DEVERR_COPY_PAIR.
 * Precondition: dst ids are distinct and no dst is also a src in the same
 * call (the block manager never produces anything else); otherwise the
 * result is undefined.  num_pairs == 0 launches nothing.
 */
int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int num_blocks,
                   pa_dtype dtype, pa_stream_t stream);

/*
 * Chunked-prefill attention: several new tokens per sequence attend over the
 * paged cache at once ("Can OS paging techniques reduce LLM serving memory
 * waste?", second paragraph: attention block by block over non-contiguous
 * blocks; "Why OS Virtual Memory Paging Saved LLM Inference: The vLLM
 * Breakthrough", section 2: the cache fills as tokens arrive).  The pages
 * describe only the single-token case; this is its causal multi-token form.
 *
 * Sequence s owns query rows query_start[s] .. query_start[s+1]-1 of q: its
 * last C_s = query_start[s+1] - query_start[s] tokens, already written to the
 * cache (pa_reshape_and_cache first, as for decode), so context_lens[s] =
 * L_s >= C_s.  Row i is the token at position L_s - C_s + i and attends to
 * positions 0 .. L_s - C_s + i:
 *   out[t, h, :] = softmax(scale * q[t, h, :] . K_s[0..p]) V_s[0..p]
 * with kv head h / (num_q_heads / num_kv_heads).
 *
 *   out          fp32 [num_tokens, num_q_heads, head_dim] (device, 16-byte aligned)
 *   q            cache dtype [num_tokens, num_q_heads, head_dim] (device, 16-byte aligned)
 *   k/v_cache    [num_blocks, num_kv_heads, block_size, head_dim] (device)
 *   block_tables int32 [num_seqs, max_blocks_per_seq] (device)
 *   context_lens int32 [num_seqs] (device), tokens including the chunk
 *   query_start  int32 [num_seqs + 1] (device), non-decreasing, query_start[0] = 0,
 *                query_start[num_seqs] = num_tokens
 *   max_query_len host upper bound of every C_s (sizes the grid; the rows of a
 *                longer chunk past what the grid covers are not computed, and
 *                PA_DEVERR_CONTEXT_LEN is set)
 * head_dim 64 or 128, block_size 16 or 32, group size up to 16, fp16 or
 * bf16.  Runs on the tensor cores (tcgen05, fp32 accumulation): Q.K^T in the
 * cache dtype; P.V in fp16 -- the softmax weights rounded to fp16 (2^-11
 * relative; the row sums add the rounded values), and a bf16 V tile converted
 * to fp16 in shared memory, which is exact for |v| <= 65504.  A bf16 V value
 * of |v| >= 65520 becomes infinite there, so the output rows of the query tile
 * that reads it come out not finite; PA_DEVERR_RANGE reports any non-finite
 * output row of a bf16 cache (non-finite q or K elements included).  No workspace,
 * nothing allocated.  A chunk longer than its
 * context, a context longer than the table, or rows outside
 * [0, num_tokens) set PA_DEVERR_CONTEXT_LEN and leave that sequence's rows
 * unwritten; block ids outside the pool are skipped and set
 * PA_DEVERR_BLOCK_ID.  Rows of a sequence whose C_s is 0 are none.
 */
int pa_paged_prefill_attention(float *out, const void *q, const void *k_cache,
                               const void *v_cache, const int32_t *block_tables,
                               const int32_t *context_lens, const int32_t *query_start,
                               float scale, int num_kv_heads, int num_seqs, int num_tokens,
                               int num_q_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, int max_query_len, int num_blocks,
                               pa_dtype dtype, pa_stream_t stream);

/*
 * Read the sticky device error word of the current device into *flags
 * (PA_DEVERR_* bits; may be NULL), clearing it if `clear` is non-zero.
 * Synchronises the device.  Returns PA_OK when no bit is set,
 * PA_ERR_DEVICE_BOUNDS when one is, PA_ERR_CUDA on a CUDA failure.
 */
int pa_device_error(unsigned *flags, int clear);

/* ------------------------------------------------------------------------
 * Host block manager: free list, reference counts, fork, copy-on-write.
 * ([P1] section 2: blocks allocated one by one as tokens arrive; [P1]
 * section 3: branches share prompt blocks, a writing branch gets a private
 * block; [P3] second paragraph: a KV cache manager keeps a block table per
 * request.)  Pure host C++; no CUDA call.  Not thread-safe: one manager per
 * thread or external locking.
 *
 * Policy: the free list is first-in-first-out, initialised from free_order
 * (NULL = 0 .. num_blocks-1); blocks whose reference count drops to zero go
 * to its back (a prefix-cache hit may take a block out of its middle).
 * Every failing call returns a negative pa_status and leaves the manager
 * unchanged.
 * ---------------------------------------------------------------------- */
typedef struct pa_bm pa_bm;

/* NULL on bad arguments (num_blocks < 0, block_size <= 0, free_order not a
 * permutation of 0 .. num_blocks-1). */
pa_bm *pa_bm_create(int num_blocks, int block_size, const int32_t *free_order);
void pa_bm_destroy(pa_bm *bm);

/* New sequence holding num_tokens (>= 0) prompt tokens: takes
 * ceil(num_tokens / block_size) blocks and, if slots_out is not NULL, writes
 * the num_tokens slots (int64) in token order.  PA_ERR_SEQ if seq exists. */
int pa_bm_allocate(pa_bm *bm, int64_t seq, int num_tokens, int64_t *slots_out);

/* child gets a copy of parent's block table and length; every block gains a
 * reference.  PA_ERR_SEQ if parent is unknown or child exists. */
int pa_bm_fork(pa_bm *bm, int64_t parent, int64_t child);

/* Reserve the slot of the sequence's next token (position t = length):
 * a new block when t % block_size == 0; otherwise, when the last block is
 * shared, a new private block whose copy (src = old, dst = new) the caller
 * must perform before writing; otherwise the last block.  Writes the slot to
 * *slot_out; returns 1 and writes *cow_src/*cow_dst when a copy is needed,
 * 0 when not, or a negative pa_status. */
int pa_bm_append_slot(pa_bm *bm, int64_t seq, int64_t *slot_out, int32_t *cow_src,
                      int32_t *cow_dst);

/* Batched append: one pa_bm_append_slot per entry of seqs[0..n), in order.
 * slots_out int64 [n]; cow_pairs_out int64 [n, 2] receives the copy pairs in
 * order of occurrence, *num_cow_out their count.  All-or-nothing: on failure
 * every append of the batch is undone. */
int pa_bm_append_slots(pa_bm *bm, const int64_t *seqs, int n, int64_t *slots_out,
                       int64_t *cow_pairs_out, int *num_cow_out);

/* Drop the sequence: one reference less on each of its blocks.  A block
 * that reaches zero goes to the back of the free list; if it holds a cached
 * prompt prefix (pa_bm_allocate_prefix) it stays in the cache until the free
 * list hands it out again. */
int pa_bm_free(pa_bm *bm, int64_t seq);

/*
 * Prefix caching across requests ([P3] second paragraph: blocks may be
 * shared across the requests of a batch; [P2] introduction and "From
 * Contiguous Reserves to Paged KV Blocks": block tables make KV memory
 * reusable and shareable).  The pages give no mechanism; the one here:
 *
 * A block that a prompt fills completely is identified by its whole token
 * prefix tokens[0 .. (j+1)*block_size) (compared exactly, never by hash
 * alone).  New sequence `seq` with the prompt tokens[0 .. num_tokens)
 * (int32 token ids, host memory): its full blocks are looked up in order and
 * the lookup stops at the first prefix not cached; each hit joins the table
 * with one more reference (a cached block waiting in the free list leaves
 * it).  The remaining ceil(num_tokens / block_size) - hits blocks come from
 * the front of the free list as in pa_bm_allocate, and each of them that is
 * full is entered in the cache under its prefix (replacing an older entry
 * for the same prefix).  slots_out (int64 [num_tokens], may be NULL) gets -1
 * for the tokens of hit blocks -- their K/V are already in the pool and
 * pa_reshape_and_cache skips negative slots -- and the slot of every other
 * token; *num_cached_out (may be NULL) = hits * block_size.  Only prompt
 * blocks are entered; blocks filled later by appends are not.  Cached
 * blocks are full, so appends never write or copy them.
 *
 * A block leaves the cache when any call takes it from the free list for
 * new content.  PA_ERR_SEQ if seq exists; PA_ERR_NO_BLOCKS (nothing
 * changed) if the free list, less the hits it holds, is too short.
 */
int pa_bm_allocate_prefix(pa_bm *bm, int64_t seq, const int32_t *tokens, int num_tokens,
                          int64_t *slots_out, int *num_cached_out);
/* Number of blocks entered in the prefix cache (held or free). */
int pa_bm_num_cached(const pa_bm *bm);

/* Copy the sequence's block table into out[0 .. cap) (*n_out = its length);
 * PA_ERR_ARG if cap is too small. */
int pa_bm_block_table(const pa_bm *bm, int64_t seq, int32_t *out, int cap, int *n_out);

/* Block tables of n sequences as one int32 [n, cap] array padded with -1,
 * and their lengths (int32 [n], may be NULL). */
int pa_bm_block_tables(const pa_bm *bm, const int64_t *seqs, int n, int32_t *out, int cap,
                       int32_t *lens_out);

/* Token count of the sequence (or a negative pa_status). */
int pa_bm_seq_len(const pa_bm *bm, int64_t seq);
int pa_bm_num_free(const pa_bm *bm);
/* Reference count of a block (or PA_ERR_ARG). */
int pa_bm_ref_count(const pa_bm *bm, int32_t block);
/* Number of live sequences. */
int pa_bm_num_seqs(const pa_bm *bm);

/*
 * KV memory accounting of the pool ([P1] section 1 "The Contiguous
 * Allocation Problem" and section 3: paged blocks leave idle only the tail of
 * each sequence's last block, and shared prompt blocks are stored once).
 *   used_blocks    distinct blocks held by some sequence
 *   shared_blocks  blocks held by more than one sequence
 *   logical_tokens sum of the sequences' lengths (shared tokens counted per holder)
 *   filled_slots   sum over used blocks of the largest fill any holder gives it
 * The idle slots are used_blocks * block_size - filled_slots.
 */
typedef struct {
  int64_t num_blocks, free_blocks, used_blocks, shared_blocks;
  int64_t num_seqs, logical_tokens, filled_slots, block_size;
} pa_bm_stats_t;
int pa_bm_stats(const pa_bm *bm, pa_bm_stats_t *out);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
