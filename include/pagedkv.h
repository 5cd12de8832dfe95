/*
 * pagedkv.h -- C ABI of the B200 paged-KV decode library (libpagedkv.so).
 *
 * Three GPU operations form the decode hot path of a paged KV cache:
 *
 *   paged_attention_decode   one query token per head attends over a KV cache held
 *                            in fixed-size physical blocks, found through a
 *                            per-sequence block table;
 *   reshape_and_cache        each new token's K/V row is written into its slot;
 *   copy_blocks              whole blocks are copied for copy-on-write.
 *
 * A host block manager (bm_*) hands out the physical blocks, slots and
 * copy-on-write pairs that these operations consume; it is not on the GPU path.
 *
 * Conventions shared by every GPU entry point
 * -------------------------------------------
 *  - Every buffer is owned by the caller; the library allocates nothing of its
 *    own on the GPU.  Pointers marked "device" must be device memory of the
 *    current CUDA device; "host" pointers are ordinary host memory.
 *  - fp16 means IEEE 754 binary16; the buffers are typed void* so that this
 *    header needs no CUDA include.  fp16 buffers must be 16-byte aligned.
 *  - KV pool layout: key_cache and value_cache are each
 *        [num_blocks][num_kv_heads][block_size][head_dim]  fp16, contiguous,
 *    so the rows of one (block, kv head) are one contiguous tile.  The pages
 *    only say a block holds "block_size x num_kv_heads x head_dim" values
 *    (lpnh.cn/news/2758356 §2.1); the head-major order inside a block is this
 *    library's choice.
 *  - A flat slot s addresses row s % block_size of physical block
 *    s / block_size.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  The GPU
 *    calls only enqueue work and return; they never synchronize.
 *  - Return value: PAGEDKV_OK (0) or a negative PAGEDKV_E* code; nothing is
 *    enqueued when an argument is rejected.  pagedkv_last_error() returns a
 *    message for the calling thread's last failure.  No call throws.
 *  - Values that live on the device cannot be checked before launch.  The
 *    kernels check them (block ids, context lengths, slots) and, instead of
 *    faulting, skip the bad access and set a bit in a per-device error word
 *    that pagedkv_device_errors() reads.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PAGEDKV_API __attribute__((visibility("default")))
#else
#define PAGEDKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes --------------------------------------------------------- */
#define PAGEDKV_OK 0
#define PAGEDKV_EINVAL (-1)       /* invalid argument (null, misaligned, out of range) */
#define PAGEDKV_EUNSUPPORTED (-2) /* shape outside the supported set */
#define PAGEDKV_ECUDA (-3)        /* CUDA runtime or launch error */
#define PAGEDKV_EWORKSPACE (-4)   /* workspace missing or smaller than required */
#define PAGEDKV_ENOMEM (-5)       /* block pool exhausted (block manager) */
#define PAGEDKV_ENOENT (-6)       /* unknown sequence id (block manager) */
#define PAGEDKV_ERANGE (-7)       /* caller's output buffer too small */

/* ---- bits of the per-device error word ------------------------------------ */
#define PAGEDKV_DEVERR_BLOCK_ID 1u    /* a block id outside [0, num_blocks): block 0 read instead */
#define PAGEDKV_DEVERR_CONTEXT_LEN 2u /* a context length <= 0 (output zeros) or beyond
                                         max_context_len / the table (clamped) */
#define PAGEDKV_DEVERR_SLOT 4u        /* a slot beyond the pool: that token was skipped */
#define PAGEDKV_DEVERR_TIMEOUT 8u     /* a pipeline wait gave up after ~2 s; output invalid */
#define PAGEDKV_DEVERR_INTERNAL 16u   /* a kernel found its launch set-up inconsistent (did
                                         nothing), or a workspace's work counters did not
                                         start at zero (outputs invalid) */
#define PAGEDKV_DEVERR_PREFIX 32u     /* a shared-prefix group or prefix length was inconsistent,
                                         or a host bound on the prefix / suffix lengths was below
                                         a real length: the affected outputs are invalid */

/* Message of the calling thread's last failed call ("" if none). */
PAGEDKV_API const char *pagedkv_last_error(void);

/* Reads (and, if clear != 0, zeroes) the error word of the current device.
 * Synchronizes the device first.  Returns PAGEDKV_OK or PAGEDKV_ECUDA. */
PAGEDKV_API int pagedkv_device_errors(unsigned int *flags, int clear);

/* Self-test of the failure path every kernel pipeline uses.  Enqueues a kernel
 * that waits on a barrier nothing completes, with the same bounded wait as the
 * attention kernels, for timeout_us microseconds (1 .. 1e6); the wait then
 * gives up, sets PAGEDKV_DEVERR_TIMEOUT in the error word and the kernel
 * returns normally.  It never faults and never hangs, and the device stays
 * usable.  Read the result with pagedkv_device_errors.  Errors: EINVAL, ECUDA. */
PAGEDKV_API int pagedkv_selftest_wait_timeout(unsigned int timeout_us, void *stream);

/* ---- paged decode attention ------------------------------------------------
 *
 * For every sequence b < num_seqs and query head h < num_heads, with
 * G = num_heads / num_kv_heads and kv head kvh = h / G (contiguous groups):
 *
 *     K_b[i] = key_cache  [block_tables[b][i / bs]][kvh][i % bs][:]   for i < L_b
 *     V_b[i] = value_cache[block_tables[b][i / bs]][kvh][i % bs][:]
 *     out[b][h][:] = softmax_i(scale * q[b][h][:] . K_b[i]) . V_b
 *
 * where L_b = context_lens[b] counts every cached token including the one
 * written this step.  The attention reads each sequence's K/V through its block
 * table (the attention looks up each block through the table while it runs:
 * lpnh.cn/news/1824136 §2.2 item 3 and §3.2 step 4; the table itself: 5688vip ch. 4 "PagedAttention：显存管理、分页机制、
 * 块大小选择", section "分页机制：块表与物理块的组织方式"; lpnh.cn/news/2758356 §2.2).
 * Accumulation is fp32; out is rounded once to fp16 (round to nearest even).
 *
 *   out            device fp16 [num_seqs][num_heads][head_dim]
 *   q              device fp16 [num_seqs][num_heads][head_dim]
 *   key_cache,
 *   value_cache    device fp16 [num_blocks][num_kv_heads][block_size][head_dim]
 *   block_tables   device int32 [num_seqs][max_blocks_per_seq]; entries at and
 *                  beyond ceil(L_b / block_size) are never read
 *   context_lens   device int32 [num_seqs], 1 <= L_b <= max_context_len
 *   scale          multiplies q.K (usually 1/sqrt(head_dim))
 *   head_dim       64 or 128;  block_size 4, 8, 16, 32 or 64
 *   num_heads      a multiple of num_kv_heads
 *   max_context_len  an upper bound of every L_b, <= max_blocks_per_seq * block_size
 *   partition_size 0 = chosen by the library; -1 = single pass; > 0 = split each
 *                  context into partitions of this many tokens (a multiple of 16
 *                  and of block_size), computed in parallel and merged by a
 *                  second kernel.
 *   workspace      device scratch of at least paged_attention_workspace_bytes(...)
 *                  bytes (16-byte aligned); may be NULL when that function returns
 *                  0.  Its first 32 bytes are work counters (grouped queries, 2..8
 *                  query heads per kv head, take their work items from them): they
 *                  must be zero before the workspace's first use -- allocate it
 *                  zeroed or cudaMemsetAsync them once -- and every call leaves
 *                  them zero again.  A launch that finds its ticket not at zero
 *                  sets PAGEDKV_DEVERR_INTERNAL (some outputs are then invalid);
 *                  zero the counters again after that flag.  The rest holds the
 *                  split-K partial results, needs no initialization and is
 *                  garbage afterwards.
 *                  Calls that may run at the same time need separate workspaces.
 *
 * num_seqs == 0 is a no-op.  Errors: EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
PAGEDKV_API int paged_attention_decode(void *out, const void *q,
                           const void *key_cache, const void *value_cache,
                           const int32_t *block_tables, const int32_t *context_lens,
                           float scale, int block_size, int num_kv_heads,
                           int num_seqs, int num_heads, int head_dim,
                           int max_blocks_per_seq, int num_blocks, int max_context_len,
                           int partition_size, void *workspace, size_t workspace_bytes,
                           void *stream);

/* Workspace bytes paged_attention_decode needs for these arguments (0 when it
 * needs none: a single pass over one kv head per query head).  Returns 0 for
 * arguments it would reject too. */
PAGEDKV_API size_t paged_attention_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                       int head_dim, int block_size, int max_context_len,
                                       int partition_size);

/* ---- fused append + decode ----------------------------------------------------------
 *
 * One decode step in one call: each sequence's new K/V row is written into the
 * cache and the attention then reads it, as reshape_and_cache followed by
 * paged_attention_decode would (the new token scattered into its block, then
 * the block-table gather: lpnh.cn/news/1824136 §3.1 and §3.2 steps 3-4).
 *
 * The new token is position L_b - 1 of sequence b, so its slot is implied by
 * the table: row (L_b - 1) % block_size of block
 * block_tables[b][(L_b - 1) / block_size]; no slot mapping is passed.  That
 * block must belong to sequence b alone (a shared block is copied first:
 * copy_blocks), as it must for reshape_and_cache.
 *
 *   k_new, v_new   device fp16 [num_seqs][num_kv_heads][head_dim], 16-byte aligned
 *   key_cache,
 *   value_cache    as for paged_attention_decode; written at the new slots only
 *   the rest       as for paged_attention_decode (same workspace size)
 *
 * Results: out as paged_attention_decode computes it on the updated cache, and
 * the cache bytes as reshape_and_cache writes them.  A sequence whose length is
 * rejected on the device (L_b <= 0 or > max_context_len) or whose block id is
 * out of range gets no write; the error word says so.
 * num_seqs == 0 is a no-op.  Errors: EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
PAGEDKV_API int paged_attention_decode_append(void *out, const void *q,
                           const void *k_new, const void *v_new,
                           void *key_cache, void *value_cache,
                           const int32_t *block_tables, const int32_t *context_lens,
                           float scale, int block_size, int num_kv_heads,
                           int num_seqs, int num_heads, int head_dim,
                           int max_blocks_per_seq, int num_blocks, int max_context_len,
                           int partition_size, void *workspace, size_t workspace_bytes,
                           void *stream);

/* ---- shared-prefix decode -----------------------------------------------------------
 *
 * Sequences forked from one prompt (parallel sampling, beam search) or served
 * from one cached prefix reference the same physical blocks at the start of
 * their block tables (copy-on-write sharing: lpnh.cn/news/2758356 §4.1-§4.2;
 * prefix caching: n1n.ai "前缀缓存").  paged_attention_decode reads such a
 * block once per sequence; this call reads it once per group:
 *
 *   prefix pass   for every group, kv head and partition of the shared prefix,
 *                 one tensor-core tile whose columns are the members' query
 *                 heads of that kv head;
 *   suffix pass   every sequence over the rest of its context [P_b, L_b);
 *   merge         the partial softmax states of both, as split-K merges them.
 *
 * The result is paged_attention_decode's (same formula, fp32 accumulation,
 * within rounding of it).  With k_new / v_new given, the new rows are written
 * first as paged_attention_decode_append writes them (they always lie in the
 * suffix).
 *
 *   seq_prefix_tokens  device int32 [num_seqs]: P_b, the tokens of sequence b
 *                  that its group's prefix pass covers; 0 = none.  A multiple of
 *                  block_size and at most L_b - 1.  A sequence with P_b > 0 must
 *                  be a member of a group: one that no group lists is not
 *                  detected on the device (its output is then invalid);
 *                  paged_decode_step_host checks this on the host.
 *   groups         device int32 [num_groups][PAGEDKV_GROUP_WIDTH]: the group's
 *                  prefix length in blocks, then up to 8 member sequence indices
 *                  (-1 = unused).  A group may hold at most 8 / G members
 *                  (G = num_heads / num_kv_heads).  Every member's first
 *                  (prefix blocks) table entries must equal the first member's,
 *                  and its seq_prefix_tokens must be that many tokens.  A member
 *                  breaking these rules is left out of the prefix pass and sets
 *                  PAGEDKV_DEVERR_PREFIX; its output is then invalid.  May be
 *                  NULL when num_groups is 0.
 *   max_prefix_tokens, max_suffix_tokens  host upper bounds of the groups' prefix
 *                  lengths and of L_b - P_b over the batch (0 = max_context_len);
 *                  they size the launch grids.  With up to 1024 groups the prefix
 *                  pass runs on persistent CTAs that take every group's items
 *                  from a queue, so max_prefix_tokens only sizes that grid; with
 *                  more groups, and for max_suffix_tokens always, a bound below a
 *                  real length leaves that work undone and sets
 *                  PAGEDKV_DEVERR_PREFIX.  When max_suffix_tokens fits one
 *                  partition, the suffix pass folds the prefix partials into
 *                  every output itself and no merge kernel is launched.
 *   partition_size 0 or -1 = 512 tokens; else as for paged_attention_decode.
 *                  The call always splits.
 *   workspace      at least paged_attention_shared_prefix_workspace_bytes(...).
 *   the rest       as for paged_attention_decode / _append.
 *
 * Needs block_size >= 8 and G <= 8 (else EUNSUPPORTED).  pagedkv_prefix_groups
 * builds seq_prefix_tokens and groups from host copies of the tables.
 * num_seqs == 0 is a no-op.  Errors: EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
#define PAGEDKV_GROUP_WIDTH 9
#define PAGEDKV_GROUP_MAX_MEMBERS 8

PAGEDKV_API int paged_attention_decode_shared_prefix(void *out, const void *q,
                           const void *k_new, const void *v_new,
                           void *key_cache, void *value_cache,
                           const int32_t *block_tables, const int32_t *context_lens,
                           const int32_t *seq_prefix_tokens, const int32_t *groups,
                           int num_groups, int max_prefix_tokens, int max_suffix_tokens,
                           float scale, int block_size, int num_kv_heads,
                           int num_seqs, int num_heads, int head_dim,
                           int max_blocks_per_seq, int num_blocks, int max_context_len,
                           int partition_size, void *workspace, size_t workspace_bytes,
                           void *stream);

/* Workspace bytes paged_attention_decode_shared_prefix needs (0 for arguments it
 * would reject). */
PAGEDKV_API size_t paged_attention_shared_prefix_workspace_bytes(int num_seqs, int num_heads,
                           int num_kv_heads, int head_dim, int block_size,
                           int max_context_len, int partition_size);

/* Host helper: groups of a batch that share table prefixes.
 *
 * From host copies of the block tables ([num_seqs][max_blocks_per_seq], -1
 * padded) and context lengths: sequences whose tables start with the same
 * physical blocks are grouped, at most max_members (1..8; pass 8 / G) per group,
 * with prefix = the members' common leading blocks, counting only whole blocks
 * before each member's last token.  Sequences are bucketed by their first
 * block, sorted by table inside a bucket and cut in that order into groups;
 * a run with fewer than 2 members or no common block forms no group.
 *
 *   seq_prefix_tokens  host int32 [num_seqs] out: prefix blocks * block_size of
 *                      the sequence's group, 0 = none
 *   groups             host int32 [groups_capacity][PAGEDKV_GROUP_WIDTH] out
 *
 * Returns the number of groups written (>= 0), or EINVAL, or ERANGE when more
 * than groups_capacity groups exist (seq_prefix_tokens is then all 0).  A
 * capacity of num_seqs / 2 always suffices. */
PAGEDKV_API int pagedkv_prefix_groups(const int32_t *block_tables, const int32_t *context_lens,
                           int num_seqs, int max_blocks_per_seq, int block_size,
                           int max_members, int32_t *seq_prefix_tokens, int32_t *groups,
                           int groups_capacity);

/* ---- one decode step from host buffers -----------------------------------------------
 *
 * The step a serving loop runs for one attention layer, driven from host
 * memory: the block manager's tables and the step's inputs go to the GPU, the
 * new token's K/V is written into its block and the attention gathers through
 * the tables, and the output comes back (lpnh.cn/news/1824136 §3.2 steps 3-5;
 * copy-on-write before the write: lpnh.cn/news/2758356 §4.2).  Enqueued on
 * `stream`, in this order:
 *
 *   1. host -> device copies (one cudaMemcpyAsync per array) of block_tables,
 *      context_lens, the copy pairs, the shared-prefix arrays, q, k_new, v_new
 *      into the caller's staging buffer;
 *   2. copy_blocks of the pairs (if any);
 *   3. paged_attention_decode_append, or with seq_prefix_tokens_host given
 *      paged_attention_decode_shared_prefix with k_new / v_new (its grid bounds
 *      taken from the host arrays);
 *   4. a device -> host copy of the output into out_host.
 *
 * A plain step (no shared prefixes) of at least 128 sequences runs those steps
 * for up to 4 chunks of sequences, pipelined: the first chunk's inputs go up on
 * `stream`, the other chunks' on an internal copy stream; the chunks' attention
 * alternates between `stream` and an internal compute stream, each chunk
 * starting when its inputs have landed; each chunk's output comes back on an
 * internal copy stream.  The internal streams are created per host thread and
 * device at the first such call and kept until the process exits.  `stream`
 * waits for all of it, also after an error return.  Every chunk is split as
 * the whole batch would be, so the output equals that of one
 * paged_attention_decode_append call over the batch, bit for bit.
 *
 * The call returns once everything is enqueued; out_host is valid after the
 * stream synchronizes.  With pinned (page-locked) host buffers every copy is
 * asynchronous; pageable buffers work too, with copies the driver stages.
 *
 *   out_host          host fp16 [num_seqs][num_heads][head_dim]
 *   q_host            host fp16 [num_seqs][num_heads][head_dim]
 *   k_new_host,
 *   v_new_host        host fp16 [num_seqs][num_kv_heads][head_dim]: the token each
 *                     sequence appends, written at position L_b - 1
 *   block_tables_host host int32 [num_seqs][max_blocks_per_seq] (bm_build_batch)
 *   context_lens_host host int32 [num_seqs], each in [1, max_context_len]
 *                     (checked on the host: EINVAL otherwise)
 *   copy_pairs_host   host int64 [num_pairs][2] (bm_take_copies); num_pairs <=
 *                     max_pairs.  Checked on the host: ids inside the pool, no
 *                     destination repeated or used as a source (EINVAL otherwise).
 *   seq_prefix_tokens_host, groups_host, num_groups
 *                     NULL / NULL / 0 for the plain step; else host arrays as
 *                     pagedkv_prefix_groups writes them (num_groups <= num_seqs / 2);
 *                     a sequence with prefix tokens that no group lists with that
 *                     prefix length is refused (EINVAL)
 *   key_cache,
 *   value_cache       device pools as for paged_attention_decode (one layer)
 *   staging           device buffer of paged_decode_step_staging_bytes(...) bytes,
 *                     256-byte aligned, owned by the caller: the device copies of
 *                     the inputs, the output and the attention workspace.  Calls
 *                     that may run at the same time need separate staging buffers.
 *   the rest          as for paged_attention_decode_append
 *
 * num_seqs == 0 runs only the copies.  Errors: EINVAL, EUNSUPPORTED, EWORKSPACE
 * (staging too small), ECUDA (part of the step may then have been enqueued).
 */
PAGEDKV_API int paged_decode_step_host(void *out_host, const void *q_host,
                           const void *k_new_host, const void *v_new_host,
                           const int32_t *block_tables_host, const int32_t *context_lens_host,
                           const int64_t *copy_pairs_host, int num_pairs,
                           const int32_t *seq_prefix_tokens_host, const int32_t *groups_host,
                           int num_groups, void *key_cache, void *value_cache,
                           float scale, int block_size, int num_kv_heads,
                           int num_seqs, int num_heads, int head_dim,
                           int max_blocks_per_seq, int num_blocks, int max_context_len,
                           int partition_size, int max_pairs,
                           void *staging, size_t staging_bytes, void *stream);

/* Staging bytes paged_decode_step_host needs (shared_prefix != 0: for calls
 * with the shared-prefix arrays).  0 for arguments it would reject. */
PAGEDKV_API size_t paged_decode_step_staging_bytes(int num_seqs, int num_heads, int num_kv_heads,
                           int head_dim, int block_size, int max_blocks_per_seq,
                           int max_context_len, int partition_size, int max_pairs,
                           int shared_prefix);

/* The partition size paged_attention_decode uses for these arguments: the tokens
 * per split-K partition, 0 for a single pass (partition_size 0 lets the library
 * choose), or a negative PAGEDKV_E* code for arguments it would reject. */
PAGEDKV_API int paged_attention_partition_tokens(int num_seqs, int num_heads, int num_kv_heads,
                                       int head_dim, int block_size, int max_context_len,
                                       int partition_size);

/* ---- allocation-free decode ------------------------------------------------------
 *
 * The pages have no counterpart of this call; it serves callers that cannot
 * allocate device memory for a workspace: an engine that reserved nearly all
 * of HBM for its block pool at start-up, a plugin inside a runtime that owns
 * the device allocator, a latency-bound loop that cannot afford cudaMalloc /
 * cudaFree (they may synchronize the device).
 *
 * Same arguments, result and errors as paged_attention_decode, minus the
 * workspace: its scratch comes from one array compiled into the library,
 * PAGEDKV_NOALLOC_SCRATCH_BYTES (16 MiB) of device memory that every GPU
 * loading the library keeps until the process exits.  It allocates nothing
 * (no cudaMalloc, cudaFree or allocating library call).
 *  - With partition_size 0, a split the library would choose but that needs
 *    more scratch than the array holds falls back to a single pass.
 *  - A call that still needs more scratch (see paged_attention_workspace_bytes)
 *    returns PAGEDKV_EWORKSPACE and enqueues nothing.
 *  - The first call on a device that needs scratch looks up the array's device
 *    address (cudaGetSymbolAddress); make that first call before any stream
 *    capture on that device.
 *  - All calls on a device share the array and leave their partial results in
 *    it; calls that can overlap on the GPU (other streams, other threads) race.
 *    Its work counters (the first 32 bytes) are cleared at that first call's
 *    set-up (on its stream) and every call leaves them zero; nothing else needs
 *    to start at zero.
 */
#define PAGEDKV_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

PAGEDKV_API int paged_attention_decode_noalloc(void *out, const void *q,
                                               const void *key_cache, const void *value_cache,
                                               const int32_t *block_tables,
                                               const int32_t *context_lens, float scale,
                                               int block_size, int num_kv_heads, int num_seqs,
                                               int num_heads, int head_dim,
                                               int max_blocks_per_seq, int num_blocks,
                                               int max_context_len, int partition_size,
                                               void *stream);

/* ---- reshape_and_cache -------------------------------------------------------
 *
 * For every token t < num_tokens with slot s = slot_mapping[t] >= 0:
 *     key_cache  [s / bs][h][s % bs][:] = k[t][h][:]   for every kv head h
 *     value_cache[s / bs][h][s % bs][:] = v[t][h][:]
 * (the new token's K/V is scattered back into its block: lpnh.cn/news/1824136
 * §3.1; a new block is used once the last one is full: 5688vip ch. 4, section
 * "分页机制：块表与物理块的组织方式").  A slot of -1 marks padding and is
 * skipped; a slot >= num_blocks * bs is skipped and flagged
 * (PAGEDKV_DEVERR_SLOT).  Two tokens with the same slot race.
 *
 *   k, v          device fp16 [num_tokens][num_kv_heads][head_dim]
 *   key_cache,
 *   value_cache   device fp16 [num_blocks][num_kv_heads][block_size][head_dim]
 *   slot_mapping  device int64 [num_tokens]
 *   head_dim      a multiple of 8
 *
 * Bit-exact copy; num_tokens == 0 is a no-op.  Errors: EINVAL, ECUDA.
 */
PAGEDKV_API int reshape_and_cache(const void *k, const void *v, void *key_cache, void *value_cache,
                      const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                      int head_dim, int block_size, int num_blocks, void *stream);

/* ---- copy_blocks ---------------------------------------------------------------
 *
 * For every pair (src, dst) = src_dst_pairs[i] and every layer l:
 *     key_caches[l][dst] = key_caches[l][src];  value_caches[l][dst] = value_caches[l][src]
 * where a block is block_elems fp16 values (num_kv_heads * block_size * head_dim).
 * This is the copy of copy-on-write: a writer of a shared, not yet full block
 * gets a new block holding a copy of the old one (lpnh.cn/news/2758356 §4.2).
 *
 *   key_caches,
 *   value_caches   HOST arrays of num_layers device pointers, each a pool of
 *                  num_blocks blocks (16-byte aligned); num_layers <= 128
 *   src_dst_pairs  device int64 [num_pairs][2]
 *   block_elems    fp16 values per block, a multiple of 8
 *
 * Pairs must not overlap: no dst may repeat or appear as a src (one
 * bm_take_copies batch never does); overlapping pairs give unspecified block
 * contents (the CTAs copy concurrently) but stay in bounds.  An id outside [0, num_blocks) skips that pair
 * and sets PAGEDKV_DEVERR_BLOCK_ID.  Bit-exact; num_pairs == 0 is a no-op.
 * Errors: EINVAL, ECUDA.
 */
PAGEDKV_API int copy_blocks(void *const *key_caches, void *const *value_caches,
                const int64_t *src_dst_pairs, int num_pairs, int num_layers,
                size_t block_elems, int num_blocks, void *stream);

/* ---- host block manager ----------------------------------------------------------
 *
 * Free list, reference counts, on-demand growth, fork and copy-on-write, after
 * the pages' description (lpnh.cn/news/2758356 §3.1-§3.2, §4.2; the
 * PagedKVManager concept model of n1n.ai "PagedAttention 对比传统 KV 缓存",
 * section "实现逻辑代码示例"):
 *
 *  - the free list is a stack: allocation pops its last element and sets the
 *    block's refcount to 1; release pushes blocks back in table order;
 *  - a sequence grows one token at a time; a new block is taken when it has
 *    none or its last block is full;
 *  - fork makes children that share every block (refcount += children);
 *  - writing into a shared (refcount > 1) last block that is not full first
 *    copies it: a new block is taken, (src, dst) is queued for copy_blocks, the
 *    old block's refcount drops by one and the writer's entry points to the new
 *    block.  A shared full block needs no copy (the next token starts a fresh
 *    block anyway);
 *  - release decrements every block of the sequence; blocks reaching 0 return
 *    to the free list;
 *  - a queued copy has not happened yet (the pages copy the shared block
 *    before its count drops, lpnh.cn/news/2758356 §4.2, and warn that a block
 *    reclaimed early is handed out again and overwritten, §4.3): both blocks of
 *    a queued pair stay off the free list until bm_take_copies hands the pair
 *    out, even if their count reaches 0 meanwhile.  A copy-on-write of a block
 *    that is itself still waiting for its copy is queued from that block's
 *    source, so the pairs of one bm_take_copies never repeat a destination or
 *    name a destination as a source (copy_blocks' requirement).
 *
 * A failed call changes nothing.  Every call locks the manager, so reference
 * counts stay consistent when several threads share one manager (the pages
 * warn that unsynchronised counts corrupt shared blocks, lpnh.cn/news/2758356
 * §4.3).  Sequence ids are small non-negative ints; the id of a released
 * sequence is handed out again, the most recently released first, so ids stay
 * below the largest number of sequences alive at once.
 */
typedef struct pagedkv_block_manager pagedkv_block_manager;

/* free_order: host int32 [num_blocks], a permutation of 0..num_blocks-1 giving
 * the initial free list (its LAST element is handed out first); NULL means
 * 0..num_blocks-1.  Returns NULL on invalid arguments. */
PAGEDKV_API pagedkv_block_manager *bm_create(int num_blocks, int block_size, const int32_t *free_order);
PAGEDKV_API void bm_destroy(pagedkv_block_manager *bm);

/* New sequence that already holds num_tokens tokens (ceil(num_tokens/bs)
 * blocks).  Returns its id, or ENOMEM / EINVAL. */
PAGEDKV_API int bm_add_seq(pagedkv_block_manager *bm, int num_tokens);

/* Reserves the slot of the sequence's next token (allocating or copying on
 * write as described above) and stores it in *slot_out.  Returns OK, ENOMEM,
 * ENOENT or EINVAL. */
PAGEDKV_API int bm_append_token(pagedkv_block_manager *bm, int seq, int64_t *slot_out);

/* bm_append_token for seqs[0..n) in order, stopping at the first failure.
 * Returns how many succeeded (slots_out[i] valid below that), or EINVAL. */
PAGEDKV_API int bm_append_tokens(pagedkv_block_manager *bm, const int32_t *seqs, int n, int64_t *slots_out);

/* n children sharing every block of seq; their ids go to ids_out[0..n).
 * Returns OK, ENOENT or EINVAL. */
PAGEDKV_API int bm_fork(pagedkv_block_manager *bm, int seq, int n, int32_t *ids_out);

/* Releases the sequence.  Returns OK or ENOENT. */
PAGEDKV_API int bm_free_seq(pagedkv_block_manager *bm, int seq);

/* Copies the sequence's block table to out[0..n) and returns n; with out ==
 * NULL only returns n.  ERANGE if cap < n, ENOENT for an unknown id. */
PAGEDKV_API int bm_block_table(pagedkv_block_manager *bm, int seq, int32_t *out, int cap);

/* Tokens held by the sequence, or ENOENT. */
PAGEDKV_API int bm_seq_len(pagedkv_block_manager *bm, int seq);

/* Flat slots (physical block * block_size + row) of the sequence's tokens
 * first .. first+count-1, the slots reshape_and_cache writes them to (a token
 * at position i lies in row i % block_size of its table's block i / block_size:
 * 5688vip ch. 4, section "分页机制：块表与物理块的组织方式").  Returns count,
 * ENOENT, EINVAL, or ERANGE for tokens beyond the sequence's length. */
PAGEDKV_API int bm_seq_slots(pagedkv_block_manager *bm, int seq, int first, int count,
                             int64_t *slots_out);

/* Packs the tables and lengths of seqs[0..n) into block_tables[n][max_blocks]
 * (unused entries = -1) and context_lens[n].  OK, ENOENT, ERANGE or EINVAL. */
PAGEDKV_API int bm_build_batch(pagedkv_block_manager *bm, const int32_t *seqs, int n,
                   int32_t *block_tables, int max_blocks, int32_t *context_lens);

/* Moves the queued copy-on-write pairs to pairs[0..2*count) as (src, dst) and
 * returns count; with pairs == NULL only returns count.  ERANGE if cap (in
 * pairs) < count, in which case nothing is moved.  Run copy_blocks on the pairs
 * before any later write into their destinations (the next step's new rows);
 * blocks that no table references any more return to the free list here, the
 * pairs' blocks in pair order (source, then destination). */
PAGEDKV_API int bm_take_copies(pagedkv_block_manager *bm, int64_t *pairs, int cap);

/* Reference count of a block (0 = free), or EINVAL. */
PAGEDKV_API int bm_refcount(pagedkv_block_manager *bm, int block);

/* Number of free blocks. */
PAGEDKV_API int bm_num_free(pagedkv_block_manager *bm);

/* Copies the free list (bottom to top) to out and returns its length; with
 * out == NULL only returns the length.  ERANGE if cap is too small. */
PAGEDKV_API int bm_free_list(pagedkv_block_manager *bm, int32_t *out, int cap);

/* Occupancy of the pool (the utilisation and fragmentation the pages discuss:
 * tail waste per block size, 5688vip ch. 4 "块大小选择"; lpnh.cn/news/2758356
 * §5.1-§5.3).  A physical block's filled slots are the most tokens any
 * sequence referencing it keeps in it. */
typedef struct pagedkv_bm_stats {
  int64_t num_blocks;      /* pool size */
  int64_t free_blocks;     /* on the free list */
  int64_t used_blocks;     /* refcount > 0 */
  int64_t num_seqs;        /* live sequences */
  int64_t logical_tokens;  /* sum of sequence lengths (shared tokens counted per sequence) */
  int64_t filled_slots;    /* physical slots holding a token */
  int64_t allocated_slots; /* used_blocks * block_size */
  int64_t table_entries;   /* sum of table lengths (= sum of refcounts) */
  int64_t held_blocks;     /* refcount 0 but named by a queued copy pair: neither used
                              nor free until bm_take_copies */
} pagedkv_bm_stats;

/* Fills *out.  OK or EINVAL. */
PAGEDKV_API int bm_stats(pagedkv_block_manager *bm, pagedkv_bm_stats *out);

/* Message of the calling thread's last failed bm_* call ("" if none). */
PAGEDKV_API const char *bm_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
