/*
 * pkv -- paged KV-cache decode attention for NVIDIA B200 (sm_100a).
 *
 * C ABI of libpkv.so.  Plain pointers and sizes only; every device buffer is
 * owned by the caller (the library never allocates or frees device memory),
 * and every call is asynchronous on the caller's CUDA stream (`stream` is a
 * cudaStream_t passed as void*; NULL = the legacy default stream).
 *
 * Stream order: the decode kernels are programmatic dependent launches, so a
 * call's grid can be resident while the kernel before it on the stream still
 * runs.  Every read of q, the new tokens, the caches and the workspace, and
 * every write, waits for that kernel to finish.  The decode and shared-
 * prefix calls may read seq_lens, block_tables and prefix_blocks before that
 * wait, so the kernel right before such a call must not write those arrays
 * after it lets dependents launch early (griddepcontrol.launch_dependents).
 * Kernels that never do that are fine, as are copies and memsets; none of
 * this library's kernels writes them.
 *
 * The method (page titles and sections of the pages this library follows):
 *  - "vLLM 與 PagedAttention：高吞吐推理的關鍵", section 二: the KV cache is cut
 *    into fixed blocks of 16 tokens; a per-sequence block table maps logical
 *    block i to a physical block, so a logically contiguous cache can sit
 *    anywhere in memory; tables of different sequences may point at the same
 *    physical blocks (shared prefixes).
 *  - same page, section 三 (運作流程): blocks are taken on demand (step 一/二);
 *    each decoded token's K/V is written into the current block or into a new
 *    one when it is full, then attention over all earlier K/V is computed by
 *    looking them up through the block table (step 三); a finished request
 *    returns all of its blocks (step 四).
 *  - "vllm" (xiexianbin.cn), "PagedAttention 的核心原理": on-demand physical
 *    blocks, logical-to-physical block table, sharing between sequences.
 *
 * Layouts (bf16 = IEEE bfloat16, row-major, contiguous):
 *   k_cache, v_cache   [num_blocks][num_kv_heads][16][head_dim]
 *   q, out             [num_seqs][num_heads][head_dim]
 *   k, v (new tokens)  [num_tokens][num_kv_heads][head_dim]
 *   block_tables       int32 [num_seqs][max_blocks_per_seq]
 *   seq_lens           int32 [num_seqs]   tokens of each sequence, including
 *                                         the one decoded this step
 *   slot_mapping       int64 [num_tokens] slot = physical_block * 16 + offset;
 *                                         a negative slot means "skip"
 *
 * Errors: host-side argument checks return a status before anything is
 * launched.  Bad data found on the device (a table entry outside
 * [0, num_blocks), a slot past the pool, a length past the table) never
 * traps: the offending block, slot or excess length is skipped and a
 * PKV_DEV_ERR_* bit is OR-ed into *err_word when err_word (a device pointer
 * to one unsigned int) is non-NULL.  Pipeline waits inside the kernels are
 * bounded; one that gives up sets PKV_DEV_ERR_TIMEOUT instead of hanging.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#define PKV_BLOCK_TOKENS 16

typedef enum {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned buffer, bad id */
    PKV_ERR_UNSUPPORTED = 2, /* valid but not implemented (head_dim, pool size) */
    PKV_ERR_WORKSPACE = 3,   /* split-K requested without a large enough workspace */
    PKV_ERR_OOM = 4,         /* block pool exhausted (allocator state unchanged) */
    PKV_ERR_CUDA = 5         /* a CUDA runtime/driver call failed */
} pkv_status;

/* Bits OR-ed into *err_word by the kernels. */
#define PKV_DEV_ERR_BAD_SLOT 1u  /* write: slot >= num_blocks * 16, token skipped */
#define PKV_DEV_ERR_BAD_BLOCK 2u /* decode: table entry outside [0, num_blocks), block skipped */
#define PKV_DEV_ERR_BAD_LEN 4u   /* decode: seq_len < 0 or > max_blocks_per_seq * 16, clamped */
#define PKV_DEV_ERR_TIMEOUT 8u   /* a bounded pipeline wait gave up */

/* Directions of a block swap between the GPU cache and host swap space. */
#define PKV_SWAP_OUT 0 /* GPU block -> host slot */
#define PKV_SWAP_IN 1  /* host slot -> GPU block */

typedef enum {
    PKV_DECODE_AUTO = 0,    /* choose from the shapes (see pkv_paged_attention_decode) */
    PKV_DECODE_SINGLE = 1,  /* one CTA per (sequence, KV head [, group of 8 query heads]) */
    PKV_DECODE_SPLIT = 2,   /* split-K token partitions + log-sum-exp merge kernel */
    /* 3: not used (rejected with PKV_ERR_INVALID_ARG) */
    PKV_DECODE_CLUSTER = 4  /* each sequence cut into P <= 8 equal parts, one CTA each; the P
                               CTAs of a (sequence, KV head) form a thread-block cluster and
                               merge their log-sum-exp partials in distributed shared memory
                               (no workspace, no second kernel) */
} pkv_decode_variant;

/* Human-readable name of a pkv_status value (static storage). */
PKV_API const char *pkv_status_string(int status);

/* The CUDA runtime error (cudaError_t value) behind the last PKV_ERR_CUDA
 * returned on the calling thread, 0 if none yet, and its text.  Added for
 * diagnostics; the pages have no counterpart. */
PKV_API int pkv_last_cuda_error(void);
PKV_API const char *pkv_last_cuda_error_string(void);

/* Tokens per physical block (16). */
PKV_API int pkv_block_tokens(void);

/* Library version string (static storage). */
PKV_API const char *pkv_version(void);

/*
 * Cache write ("vLLM 與 PagedAttention：高吞吐推理的關鍵", section 三, step 三:
 * the new token's K/V goes into the slot the block manager handed out).
 * For every token t with slot_mapping[t] >= 0 and every KV head h:
 *   k_cache[slot / 16][h][slot % 16][:] = k[t][h][:]   (and the same for v)
 * Bit-exact copy.  head_dim must be a multiple of 8 (16-byte rows); all
 * device pointers 16-byte aligned.  Duplicate non-negative slots within one
 * call are a caller error (the surviving value is unspecified).
 * Slots >= num_blocks * 16 are skipped and flagged PKV_DEV_ERR_BAD_SLOT.
 */
PKV_API pkv_status pkv_paged_kv_write(const void *k, const void *v, void *k_cache, void *v_cache,
                              const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                              int head_dim, int64_t num_blocks, unsigned int *err_word,
                              void *stream);

/*
 * Workspace (device bytes) that the split-K variant needs for these sizes;
 * 0 if a size is invalid.  The single-pass variant needs none.
 */
PKV_API size_t pkv_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                  int max_blocks_per_seq, int partition_tokens);

/*
 * Workspace (device bytes) that `variant` can use for these sizes
 * (PKV_DECODE_AUTO: enough for any variant it may pick; PKV_DECODE_SPLIT:
 * what it needs; PKV_DECODE_SINGLE and PKV_DECODE_CLUSTER: room for the
 * optional longest-first order of the sequences, 4 bytes per sequence
 * rounded up to 256 -- they also run without any workspace); 0 if a size is
 * invalid.  partition_tokens <= 0 means 512.
 */
PKV_API size_t pkv_decode_workspace_bytes_for(int variant, int num_seqs, int num_heads,
                                              int num_kv_heads, int head_dim,
                                              int max_blocks_per_seq, int partition_tokens);

/*
 * The variant PKV_DECODE_AUTO picks for these sizes on the current device
 * given `workspace_bytes` of workspace (PKV_DECODE_SINGLE, _SPLIT or
 * _CLUSTER); -1 if a size is invalid.
 */
PKV_API int pkv_decode_variant_for(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                   int max_blocks_per_seq, int partition_tokens,
                                   size_t workspace_bytes);

/*
 * The number of parts P each sequence is cut into when `variant` runs as the
 * cluster variant: PKV_DECODE_CLUSTER gives ceil(max_blocks_per_seq * 16 /
 * partition_tokens) capped at 8; PKV_DECODE_AUTO gives its own P when it
 * picks the cluster variant for these sizes and workspace, else 0; other
 * variants 0.  -1 if a size is invalid.
 */
PKV_API int pkv_decode_cluster_parts_for(int num_seqs, int num_heads, int num_kv_heads,
                                         int head_dim, int max_blocks_per_seq, int variant,
                                         int partition_tokens, size_t workspace_bytes);

/*
 * Single-query decode attention over the paged cache (section 三, step 三:
 * attention over all earlier K/V looked up through the block table), read as
 *   out[b][h][:] = softmax_p( scale * q[b][h] . K_b[p] ) V_b[p],  p in [0, seq_lens[b])
 * where K_b[p] = k_cache[block_tables[b][p / 16]][h / (num_heads/num_kv_heads)][p % 16]
 * (query heads grouped contiguously over KV heads) and the same for V.
 * bf16 inputs, fp32 accumulation and softmax, bf16 output (round to nearest
 * even).  seq_lens[b] == 0 gives a zero row.  Table entries at or past
 * ceil(seq_lens[b] / 16) are never used: they may be read (every row holds
 * max_blocks_per_seq entries) but are never taken as block numbers.
 *
 * head_dim: 64 or 128.  num_heads % num_kv_heads == 0.  Pointers 16-byte
 * aligned.  num_blocks * num_kv_heads * 16 must be < 2^31.
 * This entry point takes PKV_DECODE_AUTO with 512-token partitions.  The
 * work units are (sequence, KV head [, group of 8 query heads]).  When they
 * fill at least 1.5 waves of the GPU at 3 CTAs per SM (4 waves if the
 * workspace cannot hold the longest-first order,
 * pkv_decode_workspace_bytes_for(PKV_DECODE_SINGLE, ...) bytes): the
 * single-pass variant.  Otherwise each sequence is cut into parts: the
 * cluster variant with P = min(8, units that fit one wave at 3 CTAs per SM /
 * units, longest table / 4 blocks) parts (P >= 2) while a part of the longest
 * sequence stays at most 64 blocks;
 * else split-K when a sequence may span more than one partition and
 * `workspace` holds pkv_decode_workspace_bytes(...) bytes; else the cluster
 * variant (P >= 2) or the single pass.  pkv_decode_variant_for() and
 * pkv_decode_cluster_parts_for() report the choice.
 * The workspace is scratch owned by the caller; calls that share one
 * workspace must be ordered on the GPU (the same stream, or events).
 */
PKV_API pkv_status pkv_paged_attention_decode(void *out, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *block_tables,
                                      int max_blocks_per_seq, const int32_t *seq_lens,
                                      int num_seqs, int num_heads, int num_kv_heads,
                                      int head_dim, int64_t num_blocks, float scale,
                                      void *workspace, size_t workspace_bytes,
                                      unsigned int *err_word, void *stream);

/*
 * As pkv_paged_attention_decode, with the variant and the split-K partition
 * length chosen by the caller.  partition_tokens: a multiple of 16 in
 * [16, 65536] (used by PKV_DECODE_SPLIT and PKV_DECODE_CLUSTER).
 * PKV_DECODE_SPLIT without enough workspace returns PKV_ERR_WORKSPACE.
 * PKV_DECODE_CLUSTER cuts every sequence into P = ceil(max_blocks_per_seq *
 * 16 / partition_tokens) (at most 8) equal parts; its workspace is optional
 * (the longest-first order when num_seqs >= 16).
 * For tuning sweeps, the environment variables PKV_DECODE_WARPS and
 * PKV_DECODE_STAGES (read at each call) pick the decode CTA shape of the
 * single-pass and split-K kernels: 4 warps x 2 ring stages (the default,
 * measured fastest), 4 x 3 or 2 x 2; other values give the default.  The
 * cluster variant always runs 4 x 2.
 */
PKV_API pkv_status pkv_paged_attention_decode_ex(void *out, const void *q, const void *k_cache,
                                         const void *v_cache, const int32_t *block_tables,
                                         int max_blocks_per_seq, const int32_t *seq_lens,
                                         int num_seqs, int num_heads, int num_kv_heads,
                                         int head_dim, int64_t num_blocks, float scale,
                                         int variant, int partition_tokens, void *workspace,
                                         size_t workspace_bytes, unsigned int *err_word,
                                         void *stream);

/*
 * One decode step with the cache write fused in: the same result as
 * pkv_paged_kv_write of k_new / v_new at each sequence's new-token slot
 * followed by pkv_paged_attention_decode_ex ("vLLM 與 PagedAttention：高吞吐推
 * 理的關鍵", section 三 step 三: write the new token's K/V, then attend over all
 * of the sequence's blocks), in one launch (two with the longest-first order
 * or the split-K merge).  k_new, v_new: [num_seqs][num_kv_heads][head_dim]
 * bf16 device, the step's new token of each sequence, which sits at position
 * seq_lens[b] - 1: its slot is block_tables[b][(len - 1) / 16] * 16 +
 * (len - 1) % 16, the slot pkv_alloc_append_token hands out.  The work unit
 * that reads a sequence's last block stores the token there before reading
 * it.  Sequences with seq_lens[b] <= 0 write nothing.  A table entry outside
 * the pool for that block is not written and is flagged
 * PKV_DEV_ERR_BAD_BLOCK.  Variants: PKV_DECODE_AUTO, _SINGLE, _SPLIT,
 * _CLUSTER.  Workspace as for
 * pkv_paged_attention_decode_ex.
 */
PKV_API pkv_status pkv_paged_decode_step(void *out, const void *q, const void *k_new,
                                         const void *v_new, void *k_cache, void *v_cache,
                                         const int32_t *block_tables, int max_blocks_per_seq,
                                         const int32_t *seq_lens, int num_seqs, int num_heads,
                                         int num_kv_heads, int head_dim, int64_t num_blocks,
                                         float scale, int variant, int partition_tokens,
                                         void *workspace, size_t workspace_bytes,
                                         unsigned int *err_word, void *stream);

/*
 * Scratch-free split-K decode.  The pages have no counterpart to this call:
 * it exists for callers that must not allocate device memory when they run
 * decode -- e.g. an engine plugin whose execution path may not allocate, a
 * server that reserves all of its memory at start-up, or code that must avoid
 * cudaMalloc/cudaFree because those can synchronise the device.
 *
 * Same arguments and result as pkv_paged_attention_decode_ex with
 * PKV_DECODE_SPLIT, minus the workspace: the split-K partials go to a
 * PKV_STATIC_SCRATCH_BYTES (32 MiB) array inside the library, which every
 * GPU that loads the library holds until the process exits.  The call itself
 * allocates nothing.
 *  - Sizes whose partials need more than PKV_STATIC_SCRATCH_BYTES (see
 *    pkv_decode_workspace_bytes) are rejected with PKV_ERR_WORKSPACE.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, once per device, with that device current).
 *  - All calls share the one array and it keeps the last call's contents
 *    (nothing in it needs clearing).  Calls that overlap on the GPU -- on
 *    unordered streams, or from several host threads -- race on it and give
 *    wrong results: order them.
 */
#define PKV_STATIC_SCRATCH_BYTES (32u << 20)
PKV_API pkv_status pkv_paged_attention_decode_static(void *out, const void *q, const void *k_cache,
                                                     const void *v_cache,
                                                     const int32_t *block_tables,
                                                     int max_blocks_per_seq,
                                                     const int32_t *seq_lens, int num_seqs,
                                                     int num_heads, int num_kv_heads,
                                                     int head_dim, int64_t num_blocks,
                                                     float scale, int partition_tokens,
                                                     unsigned int *err_word, void *stream);

/*
 * Shared-prefix ("cascade") decode -- the sharing of "vLLM 與 PagedAttention：
 * 高吞吐推理的關鍵", section 二 (無法共享: the tables of requests with a common
 * prefix point at the same physical blocks) used to cut reads: the shared
 * blocks are read once per (group, KV head) instead of once per sequence.
 * Same result as pkv_paged_attention_decode (up to fp32 rounding order).
 *
 * Groups are given in CSR form: the members of group g are the sequence
 * indices group_seqs[group_offsets[g] .. group_offsets[g+1]).  Every member b
 * of a group has prefix_blocks[b] = the number of leading blocks all members'
 * tables share (full blocks, identical entries); sequences in no group have
 * prefix_blocks[b] = 0.  The group's shared block ids are read from its first
 * member's table row.  pkv_alloc_prefix_groups builds all three arrays from
 * the allocator's state.  All five arrays are device int32.
 * Work: one launch computes each group's prefix attention in spans of 64
 * blocks (one CTA and one partial per span, its keys in steps of 64) on the
 * 5th-generation tensor cores (tcgen05.mma, queries of all members x heads
 * as the MMA rows, products in tensor memory) beside split-K
 * units (partition_tokens, <= 0: 512) that cover each sequence past its
 * prefix; a merge kernel combines the partials.  Workspace:
 * pkv_decode_prefix_workspace_bytes(...), else PKV_ERR_WORKSPACE.
 * max_suffix_blocks: an upper bound on ceil(len / 16) - prefix_blocks over the
 * batch (the blocks past each sequence's prefix), or <= 0 for "unknown"
 * (max_blocks_per_seq is used).  It sizes the suffix grid, so a tight bound
 * launches no empty partitions; a suffix longer than the bound is left
 * incomplete and flagged PKV_DEV_ERR_BAD_LEN (the bound is the caller's
 * promise, as the lengths are).
 */
PKV_API size_t pkv_decode_prefix_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                                 int max_blocks_per_seq, int partition_tokens);
PKV_API pkv_status pkv_paged_attention_decode_prefix(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
    int num_heads, int num_kv_heads, int head_dim, int64_t num_blocks, float scale,
    const int32_t *prefix_blocks, const int32_t *group_offsets, const int32_t *group_seqs,
    int num_groups, int max_suffix_blocks, int partition_tokens, void *workspace,
    size_t workspace_bytes, unsigned int *err_word, void *stream);

/*
 * The shared-prefix decode with the step's write fused in, as
 * pkv_paged_decode_step is to pkv_paged_attention_decode_ex: k_new, v_new
 * [num_seqs][num_kv_heads][head_dim] bf16 are each sequence's new token (at
 * position seq_lens[b] - 1, always past its shared prefix: the token's block
 * is private -- pkv_alloc_append_token copies a shared one first), stored by
 * the suffix unit that reads that block before it reads it.  Same cache and
 * output as pkv_paged_kv_write followed by pkv_paged_attention_decode_prefix.
 * A sequence whose prefix_blocks[b] covers its last block (the new token
 * inside the shared prefix: not what pkv_alloc_prefix_groups produces) is
 * not written and is flagged PKV_DEV_ERR_BAD_LEN.
 */
PKV_API pkv_status pkv_paged_decode_prefix_step(
    void *out, const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
    int num_heads, int num_kv_heads, int head_dim, int64_t num_blocks, float scale,
    const int32_t *prefix_blocks, const int32_t *group_offsets, const int32_t *group_seqs,
    int num_groups, int max_suffix_blocks, int partition_tokens, void *workspace,
    size_t workspace_bytes, unsigned int *err_word, void *stream);

/*
 * Block copy for copy-on-write (a sequence that shares a partly filled block,
 * e.g. a beam forked mid-block -- "vllm" (xiexianbin.cn), "PagedAttention 的核
 * 心原理": beam candidates share prefix blocks -- takes a private copy before
 * its next token is written).  For every i: all num_kv_heads x 16 slots of
 * block src[i] are copied to block dst[i], in both caches (bit copy).
 * src, dst: device int64 [n]; a dst must not be the src of another pair.
 * Ids outside [0, num_blocks) are skipped and flagged PKV_DEV_ERR_BAD_BLOCK.
 */
PKV_API pkv_status pkv_copy_blocks(void *k_cache, void *v_cache, const int64_t *src,
                                   const int64_t *dst, int n, int num_kv_heads, int head_dim,
                                   int64_t num_blocks, unsigned int *err_word, void *stream);

/*
 * Block swap between the GPU cache and host swap space (the "--swap-space"
 * of "vLLM 与 PagedAttention：大模型高性能推理服务实战", section 二 2.2: CPU
 * memory that holds the KV of preempted requests).  host_k, host_v: pinned
 * host buffers laid out like the caches, [num_host_blocks][Hkv][16][d] bf16,
 * that the device can reach (page-locked, e.g. cudaHostAlloc or torch
 * pin_memory; anything else is PKV_ERR_INVALID_ARG, checked with
 * cudaPointerGetAttributes).  For every i: direction PKV_SWAP_OUT copies GPU
 * block gpu_blocks[i] to host slot host_blocks[i]; PKV_SWAP_IN the reverse.
 * gpu_blocks, host_blocks: device-readable int64 [n] (device memory).  The
 * kernel moves the bytes itself over the host link (no staging buffer).
 * Ids out of range are skipped and flagged PKV_DEV_ERR_BAD_BLOCK.
 */
PKV_API pkv_status pkv_swap_blocks(void *k_cache, void *v_cache, void *host_k, void *host_v,
                                   const int64_t *gpu_blocks, const int64_t *host_blocks, int n,
                                   int direction, int num_kv_heads, int head_dim,
                                   int64_t num_blocks, int64_t num_host_blocks,
                                   unsigned int *err_word, void *stream);

/*
 * Paged prefill attention ("vLLM 與 PagedAttention：高吞吐推理的關鍵", section 三
 * step 二: the prompt's K/V are written into blocks, a new block taken as each
 * fills -- pkv_alloc_extend + pkv_paged_kv_write -- and the prompt attends over
 * them): causal attention of each sequence's new tokens over its paged K/V.
 * Sequence b has query rows query_start[b] .. query_start[b+1] of q / out
 * ([T][num_heads][head_dim] bf16, T = query_start[num_seqs]) and context
 * length seq_lens[b] >= its row count, including them: its new tokens sit at
 * positions seq_lens[b] - rows .. seq_lens[b] - 1 (earlier positions -- a
 * cached prefix, earlier chunks -- are read from the cache), and the token at
 * position p attends to positions [0, p].  The K/V of the new tokens must be
 * in the cache already.  max_query_len >= every sequence's row count.
 * 5th-generation tensor cores (tcgen05.mma, bf16 -> fp32 in tensor memory),
 * a persistent grid of one CTA per SM over 256-row work items, TMA-fed K and
 * V rings.
 * A sequence with seq_lens[b] < its rows or past its table is skipped
 * (rows not written) and flagged PKV_DEV_ERR_BAD_LEN; a table entry outside
 * the pool is read as zeros and flagged PKV_DEV_ERR_BAD_BLOCK.
 */
PKV_API pkv_status pkv_paged_attention_prefill(void *out, const void *q, const void *k_cache,
                                               const void *v_cache, const int32_t *block_tables,
                                               int max_blocks_per_seq, const int32_t *seq_lens,
                                               const int32_t *query_start, int num_seqs,
                                               int max_query_len, int num_heads, int num_kv_heads,
                                               int head_dim, int64_t num_blocks, float scale,
                                               unsigned int *err_word, void *stream);

/* ------------------------------------------------------------------------
 * Host block allocator (section 二 and section 三 of the first page): a pool
 * of num_blocks physical blocks with reference counts, per-sequence block
 * tables, on-demand allocation, prefix sharing by fork, and release.
 * Not thread-safe: one allocator per thread, or external locking.
 * Every failing call leaves the allocator exactly as it was.
 * ------------------------------------------------------------------------ */
typedef struct pkv_alloc pkv_alloc;

/* free_order: a permutation of [0, num_blocks) giving the initial free list
 * (blocks are taken from its front, freed blocks go to its back); NULL means
 * ascending order. */
PKV_API pkv_status pkv_alloc_create(int64_t num_blocks, const int64_t *free_order, pkv_alloc **out);
/* Releases the allocator (NULL is a no-op); the device caches are the caller's. */
PKV_API void pkv_alloc_destroy(pkv_alloc *a);

/* New sequence holding num_tokens prefilled tokens: ceil(num_tokens/16) blocks. */
PKV_API pkv_status pkv_alloc_add_seq(pkv_alloc *a, int64_t seq_id, int64_t num_tokens);

/* child gets the parent's first num_tokens tokens (num_tokens < 0: all of
 * them) by sharing the blocks that hold them; each shared block's reference
 * count goes up by one. */
PKV_API pkv_status pkv_alloc_fork(pkv_alloc *a, int64_t parent, int64_t child, int64_t num_tokens);

/* One more token for seq_id; *slot_out receives its slot.  A new block is
 * taken when the last one is full (or there is none).  Appending into a partly
 * filled last block that other tables also hold is a copy-on-write: the
 * sequence gets a fresh block in its place, and the pair (shared block, fresh
 * block) is queued for pkv_alloc_take_copies; the caller must copy those
 * blocks on the device (pkv_copy_blocks) before writing the new token. */
PKV_API pkv_status pkv_alloc_append_token(pkv_alloc *a, int64_t seq_id, int64_t *slot_out);

/* n more tokens for seq_id (a prompt or a prefill chunk), their slots into
 * slots_out [n] (host): blocks are taken as each one fills (copy-on-write
 * first if the last block is shared and partly filled); all or none. */
PKV_API pkv_status pkv_alloc_extend(pkv_alloc *a, int64_t seq_id, int64_t n, int64_t *slots_out);

/* One token for each of n distinct sequences (a decode step); all or none. */
PKV_API pkv_status pkv_alloc_append_tokens(pkv_alloc *a, const int64_t *seq_ids, int n,
                                   int64_t *slots_out);

/* pkv_alloc_append_tokens that also updates the caller's host copy of the
 * tables in place, for an engine that keeps them between steps: tables_io
 * [n][width] and lens_io [n] must hold what pkv_alloc_export gave for the same
 * seq_ids in the same order (and width) before this call, with nothing else
 * changed since.  Only the entries the step changes are written: each
 * sequence's last table entry (a new block, or the private copy that replaces
 * a shared one) and its length; a step costs O(n) instead of O(n * width).
 * A sequence whose blocks would pass width is rejected (INVALID_ARG); on any
 * error nothing changes, tables_io and lens_io included. */
PKV_API pkv_status pkv_alloc_append_tokens_into(pkv_alloc *a, const int64_t *seq_ids, int n,
                                                int64_t *slots_out, int width, int32_t *tables_io,
                                                int32_t *lens_io);

/* Takes the queued copy-on-write pairs: *n_out = their number; if cap >= it,
 * src_out[i] -> dst_out[i] are filled (host arrays) and the queue is emptied;
 * otherwise nothing is taken (call again with room for *n_out). */
PKV_API pkv_status pkv_alloc_take_copies(pkv_alloc *a, int64_t *src_out, int64_t *dst_out,
                                         int64_t cap, int64_t *n_out);

/* Host swap space of num_host_blocks slots (none by default); refused while a
 * sequence is swapped out. */
PKV_API pkv_status pkv_alloc_set_host_pool(pkv_alloc *a, int64_t num_host_blocks);

/* Preemption: move every block of seq_id to host slots (its GPU blocks return
 * to the pool; queued as PKV_SWAP_OUT pairs).  Refused with
 * PKV_ERR_UNSUPPORTED if any of its blocks is shared, PKV_ERR_OOM if the host
 * space is short.  A swapped-out sequence can only be swapped in or freed. */
PKV_API pkv_status pkv_alloc_swap_out(pkv_alloc *a, int64_t seq_id);

/* Resume: give seq_id fresh GPU blocks for its host slots (queued as
 * PKV_SWAP_IN pairs; its table then lists the new blocks).  PKV_ERR_OOM if
 * the GPU pool is short. */
PKV_API pkv_status pkv_alloc_swap_in(pkv_alloc *a, int64_t seq_id);

/* Takes the queued swap pairs of one direction: as pkv_alloc_take_copies,
 * with gpu_out[i] / host_out[i] the GPU block and host slot of pair i.  Run
 * them with pkv_swap_blocks: swap-outs before the freed GPU blocks are written
 * again, swap-ins before the sequence is decoded. */
PKV_API pkv_status pkv_alloc_take_swaps(pkv_alloc *a, int direction, int64_t *gpu_out,
                                        int64_t *host_out, int64_t cap, int64_t *n_out);

/* Release a sequence: every block whose count drops to zero returns to the pool. */
PKV_API pkv_status pkv_alloc_free_seq(pkv_alloc *a, int64_t seq_id);

/* tables_out [n][width] (entries past a sequence's blocks set to -1) and
 * lens_out [n] for the listed sequences (host memory). */
PKV_API pkv_status pkv_alloc_export(const pkv_alloc *a, const int64_t *seq_ids, int n, int width,
                            int32_t *tables_out, int32_t *lens_out);

/* free and used blocks, blocks with count > 1, and utilisation = filled
 * slots of the used blocks / (16 * used blocks) (0 when nothing is used). */
PKV_API pkv_status pkv_alloc_stats(const pkv_alloc *a, int64_t *free_blocks, int64_t *used_blocks,
                           int64_t *shared_blocks, double *utilisation);

/* The free list, front first: up to cap ids into out, the count into *n_out. */
PKV_API pkv_status pkv_alloc_free_list(const pkv_alloc *a, int64_t *out, int64_t cap, int64_t *n_out);

/* Shared-prefix groups among the listed sequences (for
 * pkv_paged_attention_decode_prefix): sequences whose first block is full and
 * held by several tables are grouped by that block (groups in order of first
 * appearance, members in list order); a group's prefix is the longest run of
 * leading blocks identical in, and full for, every member.  Outputs (host):
 * prefix_blocks_out [n] (0 outside groups), group_offsets_out [n + 1] (CSR,
 * first *num_groups_out + 1 used), group_seqs_out [n] (indices into seq_ids). */
PKV_API pkv_status pkv_alloc_prefix_groups(const pkv_alloc *a, const int64_t *seq_ids, int n,
                                           int32_t *prefix_blocks_out, int32_t *group_offsets_out,
                                           int32_t *group_seqs_out, int32_t *num_groups_out);
/* Queries (host; PKV_ERR_INVALID_ARG for an unknown id or position):
 * refcount: the number of tables holding block `block` (0 if free); seq_len:
 * the tokens of a sequence; slot_of: the cache slot (block * 16 + offset) of
 * position pos in [0, seq_len) of a sequence resident on the GPU. */
PKV_API pkv_status pkv_alloc_refcount(const pkv_alloc *a, int64_t block, int32_t *out);
PKV_API pkv_status pkv_alloc_seq_len(const pkv_alloc *a, int64_t seq_id, int64_t *len_out);
PKV_API pkv_status pkv_alloc_slot_of(const pkv_alloc *a, int64_t seq_id, int64_t pos, int64_t *slot_out);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
