// Internal launch interface between the C ABI (pkv_api.cu) and the kernels.
#pragma once

#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace pkv {

constexpr int kBlockTokens = 16;

// Maps a CUDA error to PKV_ERR_CUDA (PKV_OK for cudaSuccess) and records it
// as the calling thread's last error for pkv_last_cuda_error().
int cuda_status(cudaError_t e);

struct DecodeParams {
    __nv_bfloat16 *out;           // [B][Hq][D]
    const __nv_bfloat16 *q;       // [B][Hq][D]
    const int32_t *block_tables;  // [B][W]
    const int32_t *seq_lens;      // [B]
    float *ws_o;                  // split-K partial outputs [B][Hq][P][D] (unnormalised)
    float *ws_ml;                 // split-K partial (max, sum) [B][Hq][P][2], log2 domain
    unsigned int *err;            // nullable device error word
    long long num_blocks;
    int W;            // block-table row stride (max blocks per sequence)
    int B, Hq, Hkv;
    int group;        // Hq / Hkv
    int chunks;       // query-head chunks of <= 8 per KV head (tensor-core path)
    int part_blocks;  // blocks per CTA work unit (partition, or W for single pass)
    int num_parts;    // partitions per sequence (grid.x)
    float scale_log2; // scale * log2(e)
    // Split-K workspace addressing: partition p of a row is partial slot
    // (row * ws_parts + ws_part0 + p).  Plain split-K: ws_parts = num_parts,
    // ws_part0 = 0.
    int ws_parts, ws_part0;
    // Optional [B]: sequence b's first start_blocks[b] blocks are left out
    // (their part of the attention is computed elsewhere and merged later);
    // clamped to the sequence's full blocks.
    const int32_t *start_blocks;
    bool skip_merge;  // split-K without its merge kernel (the caller merges)
    // Optional [B]: unit z of the grid decodes sequence order[z] (longest
    // first); written by the order kernel launched just before.
    const int32_t *order;
    // Optional (the fused write + decode step): this step's new K/V
    // [B][Hkv][D], stored by the unit that holds each sequence's last block
    // into the slot of position len - 1 before that unit reads the block.
    const __nv_bfloat16 *k_new, *v_new;
    __nv_bfloat16 *k_cache, *v_cache;  // [num_blocks][Hkv][16][D], for those stores
};

// Longest-first order of the sequences (by block count) into order[B], for
// the single-pass decode grid; one CTA, counting sort.
cudaError_t launch_order(const int32_t *seq_lens, int B, int W, int32_t *order, cudaStream_t stream);

struct DecodeTuning {
    int warps;   // consumer warps per CTA
    int stages;  // TMA stages per warp (one K tile + one V tile each)
};

// Most parts of one sequence in cluster mode: the portable cluster size.
constexpr int kMaxClusterParts = 8;

// Launches the decode kernel on `stream` in one of three modes (0: single
// pass, 1: split-K + the merge kernel, 2: p.num_parts parts per sequence as
// one thread-block cluster, merged in distributed shared memory); when
// p.order is set the decode grid is launched as a programmatic dependent of
// the order kernel and waits for it.
cudaError_t launch_decode(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                          int head_dim, int mode, DecodeTuning tuning, cudaStream_t stream);

// Shared-prefix (cascade) decode: prefix blocks read once per (group, KV
// head) by a dense tensor-core kernel; suffixes by split-K; LSE merge.
constexpr int kPrefixSpanBlocks = 64;  // prefix blocks per CTA (a span: one partial per row)

struct PrefixParams {
    __nv_bfloat16 *out;
    const __nv_bfloat16 *q;
    const int32_t *block_tables;
    const int32_t *seq_lens;
    const int32_t *prefix_blocks;   // [B] shared leading blocks of each sequence (0: none)
    const int32_t *group_offsets;   // [G + 1] CSR offsets into group_seqs
    const int32_t *group_seqs;      // members of each group (sequence indices)
    float *ws_o;                    // [B][Hq][ws_parts][D]
    float *ws_ml;                   // [B][Hq][ws_parts][2]
    unsigned int *err;
    long long num_blocks;
    int W, B, Hq, Hkv, group;
    int ws_parts;      // prefix_parts + suffix partitions
    int prefix_parts;  // ceil(W / kPrefixSpanBlocks): slots 0.. hold prefix spans
    int part_blocks;   // suffix split-K partition (blocks)
    float scale_log2;
};

// One launch running prefix spans (tcgen05/TMEM) and suffix split-K units
// side by side, then the merge.  dp must describe split-K with start_blocks
// = prefix_blocks.
cudaError_t launch_cascade(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefixParams &pp,
                           const DecodeParams &dp, int head_dim, int num_groups, cudaStream_t stream);

// Causal prefill attention of each sequence's new tokens over its paged K/V.
struct PrefillParams {
    __nv_bfloat16 *out;           // [T][Hq][D]
    const __nv_bfloat16 *q;       // [T][Hq][D]
    const int32_t *block_tables;  // [B][W]
    const int32_t *seq_lens;      // [B] context length including the new tokens
    const int32_t *query_start;   // [B + 1] rows of sequence b: [query_start[b], query_start[b+1])
    unsigned int *err;
    long long num_blocks;
    int W, B, Hq, Hkv, group;
    float scale_log2;
    int items;  // work items of the persistent tcgen05 kernel (set by its launcher)
};

// On tcgen05 / TMEM: a persistent kernel, one CTA per SM, work items of two
// 128-row Q tiles.
cudaError_t launch_prefill_tc(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefillParams &p,
                              int head_dim, int max_query_len, int num_sms, cudaStream_t stream);

cudaError_t launch_copy_blocks(void *k_cache, void *v_cache, const int64_t *src, const int64_t *dst,
                               int n, int num_kv_heads, int head_dim, long long num_blocks,
                               unsigned int *err, cudaStream_t stream);

cudaError_t launch_swap_blocks(void *k_cache, void *v_cache, void *host_k, void *host_v,
                               const int64_t *gpu_blocks, const int64_t *host_blocks, int n,
                               int direction, int num_kv_heads, int head_dim, long long num_blocks,
                               long long num_host_blocks, unsigned int *err, cudaStream_t stream);

cudaError_t launch_kv_write(const void *k, const void *v, void *k_cache, void *v_cache,
                            const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                            int head_dim, long long num_blocks, unsigned int *err,
                            cudaStream_t stream);

}  // namespace pkv
