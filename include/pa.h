/*
 * pa.h -- C ABI of libpagedattn: a paged KV cache and single-query decode
 * attention over it, for NVIDIA B200 (sm_100a).
 *
 * What the pages define (cited by page title and section):
 *  [P1] "PagedAttention for professionals: how vLLM serves more requests on the
 *       same H100", sections "Beginner example: library shelves" and "The
 *       scientific explanation: why PagedAttention is a breakthrough" (+ its
 *       results list).
 *  [P2] "KV Cache and PagedAttention: Why Your LLM Server Slows Down", sections
 *       "What is the KV cache?", "How PagedAttention solves this", "How does
 *       PagedAttention work?".
 *  [P3] "The KV cache and PagedAttention: why the LLM server chokes at 10 users",
 *       the serving example and "The trade-offs".
 *  [P4] "What is PagedAttention and what did it change in LLM serving",
 *       "What is PagedAttention, simply".
 *  [P5] "KV Cache for intermediates: why long context eats the GPU and how to cut
 *       it 4x", sections "The precise scientific definition" and "The four
 *       solutions".
 * The pages describe the data structure (fixed-size blocks anywhere in one pool,
 * a per-sequence block table, on-demand growth, shared blocks with copy-on-write)
 * and the KV-size formula; they print no kernel, memory layout or attention
 * formula.  The readings taken where they are silent are stated at each call.
 *
 * Conventions for every call:
 *  - Sizes are int32 unless noted; pointers named *_host point to host memory,
 *    all other buffer pointers to device memory on the device of `stream`.
 *  - Every device buffer is owned by the caller.  The library never allocates
 *    or frees device memory.  Pool metadata (host) is owned by the pool object.
 *  - Device calls are asynchronous on `stream` (NULL = the legacy default
 *    stream).  They return PA_ERR_CUDA if the launch fails.
 *  - Arguments are checked on the host before anything is launched; a bad
 *    argument returns PA_ERR_INVALID and changes nothing.  Values that live in
 *    device memory (slots, block ids, pairs, context lengths) are checked by the
 *    kernels: an out-of-range value is skipped, never dereferenced, and its
 *    PA_DEVERR_* bit is OR-ed into *dev_error (when dev_error is non-NULL).
 *    No kernel traps.  Host-side validators for the same data are provided.
 *  - On any error, pa_last_error() returns a message (thread-local).
 *  - The pool object is not thread-safe; use one pool per thread or lock it.
 */
#ifndef PAGED_ATTN_PA_H
#define PAGED_ATTN_PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID = 1,   /* bad argument; nothing changed */
  PA_ERR_OOM = 2,       /* pool has too few free blocks; nothing changed */
  PA_ERR_NOT_FOUND = 3, /* unknown sequence id */
  PA_ERR_CUDA = 4,      /* a CUDA runtime call failed */
  PA_ERR_DEVICE = 5     /* a kernel reported PA_DEVERR_* bits (pa_check_device_error) */
} pa_status;

typedef enum pa_dtype { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

/* Bits a kernel may OR into *dev_error. */
#define PA_DEVERR_BAD_SLOT 1    /* slot_mapping entry >= num_blocks * block_size */
#define PA_DEVERR_BAD_BLOCK 2   /* block table / copy pair entry outside [0, num_blocks) */
#define PA_DEVERR_BAD_CTX 4     /* context length < 0 or > max_blocks * block_size */
#define PA_DEVERR_TIMEOUT 8     /* a bounded wait for a tile copy gave up */

/* == cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* pa_stream;

typedef struct pa_pool pa_pool;

/* ------------------------------------------------------------------------
 * Block pool (host).  [P1] "The scientific explanation": the cache is split
 * into fixed-size blocks (default 16 tokens) stored anywhere in GPU memory,
 * and a block table per request maps its logical blocks to physical ones.
 * [P1] "Beginner example": a request takes a new block only when its 17th
 * token arrives; a finished request's blocks go back to the pool and are taken
 * again at once.  [P2] "How PagedAttention solves this": on-demand pages, and
 * shared prefix pages with copy-on-write.
 * Readings: the free list is a stack (the last block freed is the first
 * reused; a fresh pool hands out 0, 1, 2, ...); growing into a partially filled
 * last block that other sequences also hold copies it first (one copy pair);
 * full shared blocks stay shared; the last holder writes in place.
 * ---------------------------------------------------------------------- */

/* Create a pool of num_blocks (>= 0) blocks of block_size (>= 1) tokens. */
pa_status pa_pool_create(int32_t num_blocks, int32_t block_size, pa_pool** pool_out);
void pa_pool_destroy(pa_pool* pool);

/* Grow sequence seq_id by n_new (>= 0) tokens, creating it if unknown.
 * slot_mapping_out_host[n_new] receives each new token's slot:
 *   physical_block * block_size + offset_in_block   (int64).
 * If the sequence's last block was partially filled and shared, it is first
 * replaced by a fresh copy: one (src, dst) pair of physical block ids is written
 * to cow_pairs_out_host[0..1] and *n_cow_out = 1 (else 0).  The caller must run
 * pa_copy_blocks on returned pairs before writing the new tokens.
 * max_cow is the capacity of cow_pairs_out_host in pairs (>= 1 if a copy can
 * happen; PA_ERR_INVALID if a copy is needed and max_cow < 1).
 * All or nothing: PA_ERR_OOM (too few free blocks) leaves the pool unchanged. */
pa_status pa_alloc(pa_pool* pool, int64_t seq_id, int32_t n_new, int64_t* slot_mapping_out_host,
                   int32_t* cow_pairs_out_host, int32_t max_cow, int32_t* n_cow_out);

/* pa_alloc for a batch: grows each of n_seqs sequences (in order; a sequence may
 * appear more than once) by n_new_each tokens, exactly as n_seqs calls of
 * pa_alloc would, in one call.  slot_mapping_out_host[n_seqs * n_new_each] is
 * sequence-major; copy pairs (at most one per sequence) go to
 * cow_pairs_out_host[2 * max_cow], their count to *n_cow_out.  All or nothing:
 * on PA_ERR_OOM, or PA_ERR_INVALID because more than max_cow pairs are needed,
 * the pool is restored exactly to its state before the call. */
pa_status pa_alloc_batch(pa_pool* pool, const int64_t* seq_ids_host, int32_t n_seqs,
                         int32_t n_new_each, int64_t* slot_mapping_out_host,
                         int32_t* cow_pairs_out_host, int32_t max_cow, int32_t* n_cow_out);

/* Drop seq_id: each of its blocks loses one holder, in logical order; a block
 * with no holder left goes on top of the free stack.  PA_ERR_NOT_FOUND if unknown. */
pa_status pa_free(pa_pool* pool, int64_t seq_id);

/* child_id becomes a copy of parent_id sharing all of its blocks ([P1] results:
 * parallel sampling with n=4 costs about the memory of n=1).
 * PA_ERR_NOT_FOUND: unknown parent; PA_ERR_INVALID: child exists. */
pa_status pa_fork(pa_pool* pool, int64_t parent_id, int64_t child_id);

/* Fine-grained eviction ([P2] "How PagedAttention solves this": under memory
 * pressure small pages move to the CPU instead of whole sequences): move
 * seq_id from pool `from` to pool `to` (e.g. a device pool and a host pool of
 * the same block size).  The sequence gets one new block in `to` per block it
 * held (logical order) and keeps its length; each old block loses one holder,
 * so a block shared with other sequences stays in `from` for them.
 * pairs_out_host[2 * max_pairs] receives the (from_block, to_block) pairs the
 * caller copies with pa_swap_blocks; *n_pairs_out their count.
 * PA_ERR_OOM: `to` has too few free blocks; PA_ERR_NOT_FOUND: unknown sequence;
 * PA_ERR_INVALID: the sequence is already in `to`, block sizes differ, or
 * max_pairs is too small.  On any error nothing changes. */
pa_status pa_swap(pa_pool* from, pa_pool* to, int64_t seq_id, int32_t* pairs_out_host,
                  int32_t max_pairs, int32_t* n_pairs_out);

/* Block-table rows for n_seqs sequences: table_out_host[i * max_blocks + j] is
 * the physical block of logical block j of seq_ids_host[i], -1 past the end;
 * ctx_lens_out_host[i] is its token count.  PA_ERR_INVALID if a sequence holds
 * more than max_blocks blocks; PA_ERR_NOT_FOUND if one is unknown. */
pa_status pa_block_table(const pa_pool* pool, const int64_t* seq_ids_host, int32_t n_seqs,
                         int32_t max_blocks, int32_t* table_out_host, int32_t* ctx_lens_out_host);

/* ------------------------------------------------------------------------
 * Prefix caching.  [P3] the serving example (the lines explained after the
 * `vllm serve` command, "--enable-prefix-caching") and "The trade-offs":
 * blocks are reused when several requests share the same beginning, such as
 * one system prompt, and the cached blocks take space in the pool; [P2] "How
 * PagedAttention solves this": shared prefix pages.  Readings (the pages give
 * no algorithm):
 *  - Only full blocks are cached, keyed by the exact token ids from the start
 *    of the sequence to the block's end (the library keys them with a 64-bit
 *    chain over (parent key, the block's ids) and compares the block's ids on
 *    every hit).  A block is keyed once it is full and every token id of its
 *    sequence up to it is known; the first block written with a key takes the
 *    entry, later copies of the same content are not entered.
 *  - Lookups happen when a sequence receives its first tokens through
 *    pa_alloc_tokens: its leading full blocks are taken from the cache while
 *    they match, but never a block that holds the last of those tokens (that
 *    token is always computed, so its K/V are written).
 *  - A cached block that loses its last holder is not freed: it joins an
 *    evictable list (a sequence's blocks in reverse logical order, so its later
 *    blocks leave first) and can still be found.  New blocks come from the
 *    free stack first, then from the oldest evictable cached block, whose entry
 *    is dropped.  pa_num_free_blocks counts both.
 *  - Sequences grown by pa_alloc / pa_alloc_batch (no token ids) stop being
 *    keyed from then on.  pa_swap carries the keying state; the moved blocks
 *    are not cached in the destination pool.
 * Off by default; turning it off returns every evictable cached block to the
 * free stack (oldest first) and drops every entry.
 * ---------------------------------------------------------------------- */
pa_status pa_pool_set_prefix_caching(pa_pool* pool, int32_t enable);

/* pa_alloc with the new tokens' ids (token_ids_host[n_new], any int32 values).
 * For a sequence that holds no token yet, with prefix caching on, the leading
 * full blocks found in the cache are shared instead of allocated: their
 * tokens get slot -1 in slot_mapping_out_host (the caller writes nothing for
 * them; pa_reshape_and_cache skips -1) and *n_cached_out = their count (a
 * multiple of block_size).  Every other token gets its slot as in pa_alloc,
 * copy-on-write pairs likewise.  Full blocks are then keyed and cached.
 * All or nothing (PA_ERR_OOM leaves the pool unchanged). */
pa_status pa_alloc_tokens(pa_pool* pool, int64_t seq_id, const int32_t* token_ids_host,
                          int32_t n_new, int64_t* slot_mapping_out_host,
                          int32_t* cow_pairs_out_host, int32_t max_cow, int32_t* n_cow_out,
                          int32_t* n_cached_out);

/* Cached blocks (held by sequences or evictable), and the evictable ones. */
int32_t pa_num_cached_blocks(const pa_pool* pool);
int32_t pa_num_evictable_blocks(const pa_pool* pool);

int32_t pa_num_free_blocks(const pa_pool* pool);
/* Number of sequences holding `block` (0 if free, -1 if out of range). */
int32_t pa_refcount(const pa_pool* pool, int32_t block);
/* Token count of seq_id, or -1 if unknown. */
int64_t pa_seq_len(const pa_pool* pool, int64_t seq_id);

/* [P5] "The precise scientific definition": KV bytes of a model =
 * 2 (key and value) x layers x tokens x kv_heads x head_dim x bytes per element. */
uint64_t pa_kv_bytes(int32_t num_layers, int64_t num_tokens, int32_t num_kv_heads,
                     int32_t head_dim, int32_t dtype_bytes);

/* ------------------------------------------------------------------------
 * Cache layout (reading; the pages fix none): one key pool and one value pool
 * per layer, each [num_blocks, num_kv_heads, block_size, head_dim] row-major in
 * `dtype`, so the (block, kv head) tile of block_size x head_dim is contiguous.
 * ---------------------------------------------------------------------- */

/* Append new tokens' keys and values to the cache ([P2] "What is the KV cache?":
 * the engine stores each token's K and V instead of recomputing them).
 * key, value: [n_tokens, num_kv_heads, head_dim] contiguous, `dtype`.
 * slot_mapping: [n_tokens] int64, device; -1 = skip the token.
 * Byte-exact copy.  An entry >= num_blocks * block_size is skipped and sets
 * PA_DEVERR_BAD_SLOT.  Duplicate slots in one call are invalid input (which copy
 * lands is unspecified).  head_dim * element size must be a multiple of 16. */
pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                               const int64_t* slot_mapping, int32_t n_tokens,
                               int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               int32_t num_blocks, pa_dtype dtype, int32_t* dev_error,
                               pa_stream stream);

/* Copy-on-write block copies ([P2] "How PagedAttention solves this").
 * k_caches_host / v_caches_host: host arrays of num_layers (1..128) device
 * pointers, one key pool and one value pool per layer.
 * pairs: [n_pairs, 2] int32 (src, dst) physical block ids, device.
 * For every pair and layer, block dst of both pools becomes a byte copy of
 * block src.  block_bytes = num_kv_heads * block_size * head_dim * element
 * size (a multiple of 16).  A dst may not appear twice and may not be a src in
 * the same call (check with pa_validate_copy_pairs); ids outside
 * [0, num_blocks) are skipped with PA_DEVERR_BAD_BLOCK. */
pa_status pa_copy_blocks(void* const* k_caches_host, void* const* v_caches_host,
                         int32_t num_layers, const int32_t* pairs, int32_t n_pairs,
                         int32_t num_blocks, int64_t block_bytes, int32_t* dev_error,
                         pa_stream stream);

/* Copy blocks between two sets of pools, e.g. a device cache and a host cache:
 * for each pair (from, to) and each layer, block `to` of dst_k / dst_v becomes a
 * byte copy of block `from` of src_k / src_v.  The four pointer arrays are host
 * arrays of num_layers (1..128) pool pointers; every pool and `pairs`
 * ([n_pairs, 2] int32) must be device memory or pinned host memory (the kernel
 * reads and writes host memory across the host link directly).
 * block_bytes = num_kv_heads * block_size * head_dim * element size (a multiple
 * of 16).  Ids outside [0, src_num_blocks) / [0, dst_num_blocks) are skipped
 * with PA_DEVERR_BAD_BLOCK. */
pa_status pa_swap_blocks(void* const* dst_k_host, void* const* dst_v_host,
                         void* const* src_k_host, void* const* src_v_host, int32_t num_layers,
                         const int32_t* pairs, int32_t n_pairs, int32_t src_num_blocks,
                         int32_t dst_num_blocks, int64_t block_bytes, int32_t* dev_error,
                         pa_stream stream);

/* ------------------------------------------------------------------------
 * Decode attention.  [P5] "The precise scientific definition": the new token
 * computes a new Q while the K and V of every earlier token must already be in
 * memory.  Reading (the pages print no formula):
 *   out[b, h, :] = sum_{j < ctx[b]} softmax_j(scale * q[b, h, :] . K_b[j, g, :]) V_b[j, g, :]
 * with g = h / (num_q_heads / num_kv_heads) ([P5] "The four solutions", GQA: a
 * group of query heads shares one K/V head; MQA is num_kv_heads = 1).  Token j
 * of batch row b is slot (block_tables[b, j / block_size], j % block_size).
 * ctx[b] counts the token the caller has just written with
 * pa_reshape_and_cache.  ctx[b] = 0 gives a zero output row.
 *
 * q, out: [batch, num_q_heads, head_dim], `dtype`; out is rounded once, to
 *   nearest even, from fp32 accumulators.
 * block_tables: [batch, max_blocks] int32, device; context_lens: [batch] int32.
 * head_dim in {64, 128}; block_size in {8, 16, 32, 64, 128}; batch <= 4096;
 * num_kv_heads <= 4096; batch * num_kv_heads <= 262144;
 * num_blocks * num_kv_heads * block_size < 2^31; num_kv_heads * max_blocks < 2^31.
 * workspace: device scratch of at least pa_decode_workspace_size(...) bytes,
 *   16-byte aligned, zero-filled once before its first use (e.g. cudaMemset);
 *   every call that completes leaves it zero-filled again, so it is reused
 *   without clearing.  Its layout does not depend on the batch or head counts:
 *   the first 256 + 4 * 262144 bytes hold counters (a 256-byte header, then one
 *   4-byte arrival count per (sequence, kv head) pair, pair b * num_kv_heads +
 *   kv_head), the rest partial results that are written before they are read.
 *   So one workspace sized for the largest group and head_dim serves calls of
 *   any batch.  After a call that reported PA_DEVERR_TIMEOUT, zero the counter
 *   bytes again.  Calls that share a workspace must be ordered on one stream.
 * The work is split across the GPU by KV blocks: 7/8 of them evenly over the
 * workers, the rest in chunks claimed by whichever workers finish first.  A
 * sequence that fits in one worker's share is done in a single pass; a longer
 * one is cut into pieces whose (max, sum, partial output) are merged with a
 * log-sum-exp combine by the worker that finishes the last piece.  One kernel
 * launch per call.
 * ---------------------------------------------------------------------- */
size_t pa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                int32_t head_dim);

pa_status pa_decode_attention(void* out, const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, const int32_t* context_lens,
                              int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                              int32_t head_dim, int32_t block_size, int32_t num_blocks,
                              int32_t max_blocks, float scale, pa_dtype dtype, void* workspace,
                              size_t workspace_bytes, int32_t* dev_error, pa_stream stream);

/* Kernel paths for pa_decode_attention_ex. */
#define PA_PATH_AUTO 0   /* tensor-core path when it applies, else the CUDA-core path */
#define PA_PATH_TC 1     /* fp16/bf16, G <= 8, block_size a multiple of 16 */
#define PA_PATH_SIMT 2   /* every supported shape and dtype */

/* Flags for pa_decode_attention_ex.
 * PA_DECODE_OVERLAP_PROLOGUE: launch the decode kernel so that its prologue runs
 * while the kernel before it on `stream` finishes (programmatic dependent
 * launch).  The prologue reads context_lens, block_tables and q; everything
 * else (the caches, out, the workspace) is touched only after the preceding
 * kernel has completed.  Use it only when that preceding kernel does not write
 * context_lens, block_tables or q -- e.g. right after pa_reshape_and_cache or
 * pa_copy_blocks, which write only the caches. */
#define PA_DECODE_OVERLAP_PROLOGUE 1

/* PA_DECODE_TEST_WAIT_EXPIRY: for tests of the failure path only, never for
 * results.  Every worker of the tensor-core kernels (pa_decode_attention_ex on
 * the tensor-core path, pa_decode_attention_int8) treats its first wait for a
 * tile as if its time limit had run out and stops; the warp that feeds it then
 * waits for the tile slot to be released, and that wait really runs out, after
 * about a second.  Each warp lets its copies in flight land before it exits.
 * The call then reports PA_DEVERR_TIMEOUT, leaves output rows of non-empty
 * contexts unwritten, and the workspace's counters must be zeroed again before
 * the next call, as after any timeout.  PA_ERR_INVALID on the CUDA-core path. */
#define PA_DECODE_TEST_WAIT_EXPIRY 0x100

/* As pa_decode_attention, with the path, the number of workers (warps that
 * split the KV blocks; 0 = automatic, else clamped to the supported range) and
 * flags chosen by the caller.  Every path and worker count gives the same result
 * up to fp32 rounding order. */
pa_status pa_decode_attention_ex(void* out, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                 int32_t num_blocks, int32_t max_blocks, float scale,
                                 pa_dtype dtype, void* workspace, size_t workspace_bytes,
                                 int32_t* dev_error, int32_t path, int32_t num_workers,
                                 int32_t flags, pa_stream stream);

/* pa_decode_attention without a caller-provided workspace.  The pages have
 * no counterpart to this call; it exists for callers that cannot allocate
 * device memory (an embedding host that hands out none, a serving loop that
 * must not call cudaMalloc while requests run, a process whose memory another
 * runtime has reserved).  The scratch is one area of 28 MiB that the library
 * declares in device memory; every GPU that loads the library holds it until
 * the process exits.  Arguments, results and errors are those of
 * pa_decode_attention, plus PA_ERR_INVALID if a shape would need more scratch
 * than the area holds: every shape whose group (num_q_heads / num_kv_heads) is
 * at most 2048 fits, larger groups may not.  Every argument is checked before
 * the device is touched.  Nothing is allocated by this call.
 * The first call on a device looks up the area's device address (once per
 * device, with that device current); make that first call before any stream
 * capture begins.  Each call first clears, on `stream`, the counters it will
 * use (256 + 4 * batch * num_kv_heads bytes at the start of the area), so a call
 * that follows one that reported PA_DEVERR_TIMEOUT starts clean.  All calls
 * share the one area, which keeps whatever the last call left in it: calls
 * whose work overlaps on the GPU (different streams, or different host threads
 * on one device) race on it and must be ordered by the caller. */
pa_status pa_decode_attention_static_ws(void* out, const void* q, const void* k_cache,
                                        const void* v_cache, const int32_t* block_tables,
                                        const int32_t* context_lens, int32_t batch,
                                        int32_t num_q_heads, int32_t num_kv_heads,
                                        int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                        int32_t max_blocks, float scale, pa_dtype dtype,
                                        int32_t* dev_error, pa_stream stream);

/* Path and worker count pa_decode_attention would use for these arguments. */
pa_status pa_decode_plan(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, pa_dtype dtype, int32_t* path_out,
                         int32_t* num_workers_out);

/* ------------------------------------------------------------------------
 * Paged prefill / chunked-prefill attention.  [P4] "What is PagedAttention,
 * simply": the prompt phase runs over the same paged cache.  Reading (the
 * pages print no formula): sequence b has n_b = query_start[b + 1] -
 * query_start[b] new tokens, the last n_b of its context_lens[b] tokens, whose
 * keys and values are already in the cache (written by pa_reshape_and_cache);
 * new token i at position p = context_lens[b] - n_b + i attends causally:
 *   out[t, h] = sum_{j <= p} softmax_j(scale q[t, h] . K_b[j, g]) V_b[j, g],
 * t = query_start[b] + i, g = h / (num_q_heads / num_kv_heads).  n_b equal to
 * the context is a whole prompt, smaller a chunk after earlier context, 1 is
 * decode.
 * q, out: [total_q, num_q_heads, head_dim], fp16 or bf16; out is rounded once
 *   from fp32 accumulators.
 * query_start: [batch + 1] int32, device, non-decreasing from 0; every n_b <=
 *   max_q (the host's bound, which sizes the launch), n_b <= context_lens[b] and
 *   query_start[b + 1] <= total_q, else the sequence is skipped (its rows of out
 *   untouched) and PA_DEVERR_BAD_CTX is set.
 * head_dim 64 or 128; num_q_heads / num_kv_heads a divisor of 64; block_size a
 * multiple of 16; batch <= 65535.  One launch.  head_dim 128 (with a group
 * dividing 128 and scale > 0) runs on the 5th-generation tensor cores (tcgen05
 * UMMA with TMEM accumulators; items of 128 (token, head) rows of one kv head,
 * K / V tiles of 128 keys; here one item per CTA, persistent through
 * pa_prefill_attention_ex with a workspace); otherwise mma.sync (64 rows per
 * CTA, 64-key tiles).  pa_prefill_attention_ex also offers the same shapes on
 * pairs of SMs (PA_PREFILL_TCGEN05_PAIR).
 * Alignment: k_cache, v_cache 16 bytes; q, out 4 (16 for the tcgen05
 * kernel, which the automatic choice then skips).  max_q * (num_q_heads /
 * num_kv_heads) < 2^31 - 256.  Errors: PA_ERR_INVALID for
 * shapes or pointers outside these limits, nothing launched.
 * ---------------------------------------------------------------------- */
pa_status pa_prefill_attention(void* out, const void* q, const void* k_cache,
                               const void* v_cache, const int32_t* block_tables,
                               const int32_t* context_lens, const int32_t* query_start,
                               int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t block_size, int32_t num_blocks,
                               int32_t max_blocks, int32_t total_q, int32_t max_q, float scale,
                               pa_dtype dtype, int32_t* dev_error, pa_stream stream);

/* Kernels for pa_prefill_attention_ex. */
#define PA_PREFILL_AUTO 0      /* the one-SM tcgen05 kernel where it applies, else mma.sync */
#define PA_PREFILL_TCGEN05 1   /* one SM per item: head_dim 128, group dividing 128,
                                  scale > 0, q and out 16-byte aligned */
#define PA_PREFILL_MMA_SYNC 2  /* every supported shape */
#define PA_PREFILL_TCGEN05_PAIR 3  /* the shapes of PA_PREFILL_TCGEN05, on pairs of SMs
                                      (clusters of two CTAs, tcgen05 cta_group::2): an item is
                                      256 rows, each SM keeps 128 of them and loads half of
                                      every key and value tile */

/* Bytes of the optional scheduling workspace of pa_prefill_attention_ex. */
#define PA_PREFILL_WORKSPACE_BYTES 16

/* pa_prefill_attention with the kernel chosen by the caller (same results up to
 * fp32 rounding order), and an optional scheduling workspace.
 * workspace: NULL, or PA_PREFILL_WORKSPACE_BYTES of device memory, 8-byte
 *   aligned, owned by the caller, zero-filled once before its first use (e.g.
 *   cudaMemset); every call leaves it zero.  With it the tcgen05 kernel is
 *   persistent (one CTA per SM taking 256-row items from a counter there: in
 *   blocks of (sequence, kv head) pairs whose keys and values fit in part of L2,
 *   the longest items first within a block), without it each
 *   CTA runs one item; the results are the same bits.  Calls sharing one workspace must not overlap on the GPU (order
 *   them on one stream).  The mma.sync kernel ignores it.
 * An unknown path, or PA_PREFILL_TCGEN05 for a shape it does not take, is
 * PA_ERR_INVALID with nothing launched. */
pa_status pa_prefill_attention_ex(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, const int32_t* query_start,
                                  int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                  int32_t max_blocks, int32_t total_q, int32_t max_q, float scale,
                                  pa_dtype dtype, int32_t* dev_error, void* workspace,
                                  int32_t path, pa_stream stream);

/* ------------------------------------------------------------------------
 * INT8 KV cache.  [P5] "The four solutions", KV-cache quantisation: keys and
 * values stored in 8 bits take about half the memory (and read bandwidth) of
 * fp16.  Scheme (reading; the pages fix none): per (token, kv head), symmetric
 * over head_dim, every step in IEEE fp32:
 *   amax = max_d |x_d|,  scale = amax / 127,
 *   code_d = round-half-to-even(x_d / scale) clamped to [-127, 127]
 * (a row of zeros has scale 0 and zero codes); an element reads back as
 * code * scale.  head_dim is 128 and block_size a multiple of 16.
 *
 * Layout: per layer a key pool and a value pool, each
 * [num_blocks, num_kv_heads, block_size / 16] records of 2112 bytes, one record
 * per 16-token group of a (block, kv head) (so a pool is
 * pa_int8_block_bytes(...) bytes per block):
 * Codes are stored offset-binary: the byte is code + 128 (code XOR 0x80).
 *   key record:   16 lines of 128 code bytes, then 16 fp32 key scales
 *                 (token order).  Group token t = 4i + 2h + e is on line
 *                 L = 2i + e + 8h; the codes of head_dim 16c .. 16c + 15 sit at
 *                 bytes L * 128 + 16 (c xor (L mod 8)) .. + 15.
 *   value record: 128 rows of 16 code bytes (row d: head_dim d of
 *                 tokens 0 .. 15 in token order), then 16 fp32 value scales.
 * Each record is what the decode kernel keeps in shared memory for one stage,
 * so one bulk copy moves it.  Block copies (copy-on-write, eviction) of an
 * INT8 cache are pa_copy_blocks / pa_swap_blocks on the two pools with
 * block_bytes = pa_int8_block_bytes(...).
 * ---------------------------------------------------------------------- */

/* Bytes of one block of one INT8 pool (0 if the shape is not supported). */
size_t pa_int8_block_bytes(int32_t num_kv_heads, int32_t head_dim, int32_t block_size);

/* Quantise new tokens into an INT8 cache: as pa_reshape_and_cache (same
 * key / value / slot_mapping arguments, `dtype` is that of key and value: f32,
 * f16 or bf16), but each (token, kv head) row is written as codes + scale by
 * the scheme above; codes and scales are bit-exact to it.  Pools and key /
 * value 16-byte aligned, slot_mapping 8.  Slots outside the pool set
 * PA_DEVERR_BAD_SLOT and are skipped; -1 is skipped silently. */
pa_status pa_reshape_and_cache_int8(const void* key, const void* value, void* k_pool,
                                    void* v_pool, const int64_t* slot_mapping, int32_t n_tokens,
                                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                    int32_t num_blocks, pa_dtype dtype, int32_t* dev_error,
                                    pa_stream stream);

/* Decode attention over an INT8 cache: the definition of pa_decode_attention
 * with K_b[j, g, :] = k_code * k_scale and V_b[j, g, :] = v_code * v_scale of
 * token j.  q and out in `dtype` (f16 or bf16); head_dim 128; group
 * (num_q_heads / num_kv_heads) <= 8; block_size in {16, 32, 64, 128}; pools
 * 16-byte aligned.  block_tables, context_lens, workspace (same size, zero-once
 * contract and reuse as pa_decode_attention), dev_error, the work split and
 * flags are those of pa_decode_attention_ex; num_workers = 0 chooses
 * automatically.  Runs on tensor cores: codes are converted exactly to fp16 /
 * bf16, products accumulate in fp32, out is rounded once. */
pa_status pa_decode_attention_int8(void* out, const void* q, const void* k_pool,
                                   const void* v_pool, const int32_t* block_tables,
                                   const int32_t* context_lens, int32_t batch,
                                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                   int32_t block_size, int32_t num_blocks, int32_t max_blocks,
                                   float scale, pa_dtype dtype, void* workspace,
                                   size_t workspace_bytes, int32_t* dev_error,
                                   int32_t num_workers, int32_t flags, pa_stream stream);

/* ------------------------------------------------------------------------
 * Host-side validators (no device work): PA_OK or PA_ERR_INVALID + message.
 * ---------------------------------------------------------------------- */
/* Every slot is -1 or in [0, num_blocks * block_size), and no slot repeats. */
pa_status pa_validate_slot_mapping(const int64_t* slot_mapping_host, int32_t n_tokens,
                                   int32_t block_size, int32_t num_blocks);
/* Each ctx in [0, max_blocks * block_size]; each of its ceil(ctx / block_size)
 * leading table entries in [0, num_blocks). */
pa_status pa_validate_block_table(const int32_t* block_tables_host,
                                  const int32_t* context_lens_host, int32_t batch,
                                  int32_t max_blocks, int32_t block_size, int32_t num_blocks);
/* Ids in range, no dst repeated, no dst also used as a src. */
pa_status pa_validate_copy_pairs(const int32_t* pairs_host, int32_t n_pairs, int32_t num_blocks);

/* Copy the device error word to the host (synchronising `stream`), then clear
 * it.  Returns PA_ERR_DEVICE with *flags_out set if any bit was set. */
pa_status pa_check_device_error(int32_t* dev_error, int32_t* flags_out, pa_stream stream);

/* Message for the last failing call on this thread ("" if none). */
const char* pa_last_error(void);

/* Number of streaming multiprocessors on the current device (0 on failure). */
int32_t pa_device_sm_count(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_ATTN_PA_H */
