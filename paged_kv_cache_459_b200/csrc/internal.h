// Internal launch interface between the C ABI (pkv_api.cu) and the kernels.
#pragma once

#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace pkv {

constexpr int kBlockTokens = 16;

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
};

struct DecodeTuning {
    int warps;   // consumer warps per CTA
    int stages;  // TMA stages per warp (one K tile + one V tile each)
};

// Balanced (stream-K) decode: a persistent grid whose warps each take an
// equal contiguous range of the flattened (sequence, head segment, block)
// tile order; segments cut between warps are merged by a second kernel.
constexpr int kStreamMaxCtasPerSm = 8;
constexpr int kStreamWarps = 4;

struct StreamParams {
    __nv_bfloat16 *out;
    const __nv_bfloat16 *q;
    const int32_t *block_tables;
    const int32_t *seq_lens;
    long long *ws_total;  // total tiles of the launch (read by the merge kernel)
    int2 *ws_dir;     // [B * Y] (first worker, last worker) of each segment
    float *ws_piece;  // [max_workers + B * Y][HP][D + 2]: o, then m[HP], then l[HP]
    unsigned int *err;
    long long num_blocks;
    long long max_workers;  // piece slots reserved for workers
    long long num_workers;  // warps of the launched grid
    int W, B, Hq, Hkv;
    int group, chunks;
    int Y;   // head segments per sequence: Hkv (one query row per KV head) or Hkv * chunks
    int HP;  // query heads per segment slot: 1, or min(8, group)
    float scale_log2;
};

cudaError_t launch_decode_stream(const CUtensorMap &tmk, const CUtensorMap &tmv,
                                 const StreamParams &p, int head_dim, cudaStream_t stream);

// Launches the decode kernel (and the merge kernel when split) on `stream`.
cudaError_t launch_decode(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                          int head_dim, bool split, DecodeTuning tuning, cudaStream_t stream);

cudaError_t launch_kv_write(const void *k, const void *v, void *k_cache, void *v_cache,
                            const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                            int head_dim, long long num_blocks, unsigned int *err,
                            cudaStream_t stream);

}  // namespace pkv
