// C ABI of libpkv.so: argument checks, TMA descriptor set-up and dispatch.
// Nothing here allocates device memory; every launch goes on the caller's
// stream.  See include/pkv.h for the contract of each entry point.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <mutex>

#include <cudaTypedefs.h>

#include "../../include/pkv.h"
#include "internal.h"

namespace {

constexpr int kDefaultPartitionTokens = 512;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// One cache array seen by TMA as a 2-D bf16 tensor: rows = (block, kv head,
// token) flattened, columns = head_dim.  Boxes are [16 rows][64 columns] --
// 128-byte rows, the 128-byte swizzle -- so a (block, head) tile of K or V is
// head_dim/64 boxes.
bool encode_cache_map(CUtensorMap *m, const void *cache, int64_t rows, int head_dim) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * 2};
    cuuint32_t box[2] = {64, 16};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(cache), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int env_int(const char *name, int fallback) {
    const char *s = std::getenv(name);
    return (s && *s) ? std::atoi(s) : fallback;
}

// The CUDA error behind the last PKV_ERR_CUDA returned on this thread.
thread_local int g_last_cuda_error = 0;

pkv_status cuda_status(cudaError_t e) { return static_cast<pkv_status>(pkv::cuda_status(e)); }

// Streaming multiprocessors of the current device (148 on B200).
int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

int num_parts_for(int max_blocks_per_seq, int partition_tokens) {
    const int pb = partition_tokens / PKV_BLOCK_TOKENS;
    return (max_blocks_per_seq + pb - 1) / pb;
}

}  // namespace

int pkv::cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return PKV_OK;
    g_last_cuda_error = static_cast<int>(e);
    return PKV_ERR_CUDA;
}

extern "C" {

int pkv_last_cuda_error(void) { return g_last_cuda_error; }

const char *pkv_last_cuda_error_string(void) {
    return cudaGetErrorString(static_cast<cudaError_t>(g_last_cuda_error));
}

const char *pkv_status_string(int status) {
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID_ARG: return "invalid argument";
        case PKV_ERR_UNSUPPORTED: return "unsupported";
        case PKV_ERR_WORKSPACE: return "workspace missing or too small";
        case PKV_ERR_OOM: return "out of blocks";
        case PKV_ERR_CUDA: return "CUDA error";
        default: return "unknown status";
    }
}

int pkv_block_tokens(void) { return PKV_BLOCK_TOKENS; }

const char *pkv_version(void) { return "pkv 0.1 sm_100a"; }

pkv_status pkv_paged_kv_write(const void *k, const void *v, void *k_cache, void *v_cache,
                              const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                              int head_dim, int64_t num_blocks, unsigned int *err_word,
                              void *stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 8 || num_blocks <= 0)
        return PKV_ERR_INVALID_ARG;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_ERR_INVALID_ARG;
    if (num_blocks > (INT64_MAX / PKV_BLOCK_TOKENS) / num_kv_heads / head_dim)
        return PKV_ERR_INVALID_ARG;
    cudaError_t e = pkv::launch_kv_write(k, v, k_cache, v_cache, slot_mapping, num_tokens,
                                         num_kv_heads, head_dim, num_blocks, err_word,
                                         static_cast<cudaStream_t>(stream));
    return cuda_status(e);
}

pkv_status pkv_copy_blocks(void *k_cache, void *v_cache, const int64_t *src, const int64_t *dst,
                           int n, int num_kv_heads, int head_dim, int64_t num_blocks,
                           unsigned int *err_word, void *stream) {
    if (n < 0 || n > 65535 || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 8 || num_blocks <= 0)
        return PKV_ERR_INVALID_ARG;
    if (n == 0) return PKV_OK;
    if (!k_cache || !v_cache || !src || !dst || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_ERR_INVALID_ARG;
    cudaError_t e = pkv::launch_copy_blocks(k_cache, v_cache, src, dst, n, num_kv_heads, head_dim,
                                            num_blocks, err_word, static_cast<cudaStream_t>(stream));
    return cuda_status(e);
}

// Device address of pinned, device-mapped host memory, or nullptr.
static void *mapped_host_pointer(void *p) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();  // clear the error the query left behind
        return nullptr;
    }
    if (attr.type != cudaMemoryTypeHost || attr.devicePointer == nullptr) return nullptr;
    return attr.devicePointer;
}

pkv_status pkv_swap_blocks(void *k_cache, void *v_cache, void *host_k, void *host_v,
                           const int64_t *gpu_blocks, const int64_t *host_blocks, int n,
                           int direction, int num_kv_heads, int head_dim, int64_t num_blocks,
                           int64_t num_host_blocks, unsigned int *err_word, void *stream) {
    if (n < 0 || n > 65535 || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 8 ||
        num_blocks <= 0 || num_host_blocks <= 0 ||
        (direction != PKV_SWAP_OUT && direction != PKV_SWAP_IN))
        return PKV_ERR_INVALID_ARG;
    if (n == 0) return PKV_OK;
    if (!k_cache || !v_cache || !host_k || !host_v || !gpu_blocks || !host_blocks ||
        !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(host_k) || !aligned16(host_v))
        return PKV_ERR_INVALID_ARG;
    void *dk = mapped_host_pointer(host_k);
    void *dv = mapped_host_pointer(host_v);
    if (!dk || !dv || !aligned16(dk) || !aligned16(dv)) return PKV_ERR_INVALID_ARG;
    cudaError_t e = pkv::launch_swap_blocks(k_cache, v_cache, dk, dv, gpu_blocks, host_blocks, n,
                                            direction, num_kv_heads, head_dim, num_blocks,
                                            num_host_blocks, err_word,
                                            static_cast<cudaStream_t>(stream));
    return cuda_status(e);
}

size_t pkv_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                  int max_blocks_per_seq, int partition_tokens) {
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || max_blocks_per_seq <= 0) return 0;
    if (partition_tokens <= 0) partition_tokens = kDefaultPartitionTokens;
    if (partition_tokens % PKV_BLOCK_TOKENS) return 0;
    const size_t parts = static_cast<size_t>(num_parts_for(max_blocks_per_seq, partition_tokens));
    const size_t rows = static_cast<size_t>(num_seqs) * num_heads * parts;
    return rows * (static_cast<size_t>(head_dim) + 2) * sizeof(float);
}

namespace {

size_t order_bytes(int num_seqs) {
    return (static_cast<size_t>(num_seqs) * sizeof(int32_t) + 255) / 256 * 256;
}

// (sequence, KV head [, group of 8 query heads]) work units of one decode.
int64_t decode_units(int num_seqs, int num_heads, int num_kv_heads) {
    return static_cast<int64_t>(num_seqs) * num_kv_heads * ((num_heads / num_kv_heads + 7) / 8);
}

// Cluster variant, automatic: as many parts per sequence as keep the whole
// grid resident at once (three CTAs per SM) -- a part that waits for a peer
// still queued would hold its slot idle; measured: 8 parts at batch 32 ran 2x
// slower than the single pass -- at most kMaxClusterParts, and at least one
// block per consumer warp (4) in a part of the longest sequence.
int cluster_parts_auto(int64_t units, int max_blocks_per_seq) {
    const int64_t slots = 3 * static_cast<int64_t>(sm_count());
    int64_t parts = slots / std::max<int64_t>(units, 1);
    parts = std::min<int64_t>(parts, pkv::kMaxClusterParts);
    parts = std::min<int64_t>(parts, std::max(1, max_blocks_per_seq / 4));
    return static_cast<int>(std::max<int64_t>(parts, 1));
}

// Cluster variant, explicit: the longest sequence cut into partition_tokens
// pieces, at most kMaxClusterParts.
int cluster_parts_for(int max_blocks_per_seq, int partition_tokens) {
    return std::min(num_parts_for(max_blocks_per_seq, partition_tokens), pkv::kMaxClusterParts);
}

// A cluster part longer than this (blocks of the longest sequence) leaves too
// few CTAs for a long context: split-K with the merge kernel balances better.
constexpr int kClusterMaxPartBlocks = 64;

struct DecodePlan {
    int variant;  // PKV_DECODE_SINGLE, _SPLIT or _CLUSTER
    int parts;    // cluster parts per sequence (cluster variant)
};


// The automatic choice.  Single pass, its units run longest first when the
// workspace holds the order (measured best when the units fill the GPU);
// when one pass would leave the GPU short of CTAs -- fewer than ~1.5 waves of
// units at 3 CTAs per SM (4 waves without the order, whose tail is longer) --
// each sequence is cut into parts: one cluster of up to 8 CTAs per unit,
// merged on chip, while a part stays short (kClusterMaxPartBlocks), else
// 512-token split-K partitions and the merge kernel (long contexts).
DecodePlan plan_auto(int num_seqs, int num_heads, int num_kv_heads, int max_blocks_per_seq,
                     int partition_tokens, size_t workspace_bytes, size_t split_bytes) {
    const int64_t units = decode_units(num_seqs, num_heads, num_kv_heads);
    const bool ordered = workspace_bytes >= order_bytes(num_seqs);
    const int64_t min_units = ordered ? 3 * 3 * sm_count() / 2 : 4 * 3 * sm_count();
    if (units >= min_units) return {PKV_DECODE_SINGLE, 1};
    const int parts = cluster_parts_auto(units, max_blocks_per_seq);
    const bool short_parts = (max_blocks_per_seq + parts - 1) / parts <= kClusterMaxPartBlocks;
    if (parts >= 2 && short_parts) return {PKV_DECODE_CLUSTER, parts};
    if (max_blocks_per_seq > partition_tokens / PKV_BLOCK_TOKENS && workspace_bytes >= split_bytes)
        return {PKV_DECODE_SPLIT, 1};
    if (parts >= 2) return {PKV_DECODE_CLUSTER, parts};
    return {PKV_DECODE_SINGLE, 1};
}

}  // namespace

size_t pkv_decode_workspace_bytes_for(int variant, int num_seqs, int num_heads, int num_kv_heads,
                                      int head_dim, int max_blocks_per_seq, int partition_tokens) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads ||
        head_dim <= 0 || max_blocks_per_seq <= 0)
        return 0;
    if (partition_tokens <= 0) partition_tokens = kDefaultPartitionTokens;
    const size_t split = pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim,
                                                    max_blocks_per_seq, partition_tokens);
    const size_t order = order_bytes(num_seqs);
    switch (variant) {
        case PKV_DECODE_SINGLE:   // optional: longest-first scheduling
        case PKV_DECODE_CLUSTER: return order;
        case PKV_DECODE_SPLIT: return split;
        case PKV_DECODE_AUTO: return std::max(split, order);
        default: return 0;
    }
}

int pkv_decode_variant_for(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                           int max_blocks_per_seq, int partition_tokens, size_t workspace_bytes) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads ||
        head_dim <= 0 || max_blocks_per_seq <= 0)
        return -1;
    if (partition_tokens <= 0) partition_tokens = kDefaultPartitionTokens;
    if (partition_tokens % PKV_BLOCK_TOKENS) return -1;
    const size_t split = pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim,
                                                    max_blocks_per_seq, partition_tokens);
    return plan_auto(num_seqs, num_heads, num_kv_heads, max_blocks_per_seq, partition_tokens,
                     workspace_bytes, split)
        .variant;
}

int pkv_decode_cluster_parts_for(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                 int max_blocks_per_seq, int variant, int partition_tokens,
                                 size_t workspace_bytes) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads ||
        head_dim <= 0 || max_blocks_per_seq <= 0)
        return -1;
    if (partition_tokens <= 0) partition_tokens = kDefaultPartitionTokens;
    if (partition_tokens % PKV_BLOCK_TOKENS) return -1;
    if (variant == PKV_DECODE_CLUSTER) return cluster_parts_for(max_blocks_per_seq, partition_tokens);
    if (variant != PKV_DECODE_AUTO) return 0;
    const size_t split = pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim,
                                                    max_blocks_per_seq, partition_tokens);
    const DecodePlan plan = plan_auto(num_seqs, num_heads, num_kv_heads, max_blocks_per_seq,
                                      partition_tokens, workspace_bytes, split);
    return plan.variant == PKV_DECODE_CLUSTER ? plan.parts : 0;
}

static pkv_status decode_impl(void *out, const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *block_tables, int max_blocks_per_seq,
                              const int32_t *seq_lens, int num_seqs, int num_heads,
                              int num_kv_heads, int head_dim, int64_t num_blocks, float scale,
                              int variant, int partition_tokens, void *workspace,
                              size_t workspace_bytes, unsigned int *err_word, void *stream,
                              const void *k_new, const void *v_new) {
    if (num_seqs < 0 || num_seqs > 65535 || num_heads <= 0 || num_kv_heads <= 0 ||
        num_heads % num_kv_heads || max_blocks_per_seq <= 0 || num_blocks <= 0 ||
        !std::isfinite(scale))
        return PKV_ERR_INVALID_ARG;
    if (variant != PKV_DECODE_AUTO && variant != PKV_DECODE_SINGLE && variant != PKV_DECODE_SPLIT &&
        variant != PKV_DECODE_CLUSTER)
        return PKV_ERR_INVALID_ARG;
    if (partition_tokens <= 0) partition_tokens = kDefaultPartitionTokens;
    if (partition_tokens % PKV_BLOCK_TOKENS || partition_tokens > 65536) return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens) return PKV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_ERR_INVALID_ARG;
    const int64_t rows = num_blocks * num_kv_heads * PKV_BLOCK_TOKENS;
    if (num_blocks > INT32_MAX / PKV_BLOCK_TOKENS / num_kv_heads) return PKV_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(max_blocks_per_seq) * PKV_BLOCK_TOKENS > INT32_MAX)
        return PKV_ERR_INVALID_ARG;

    const int part_blocks = partition_tokens / PKV_BLOCK_TOKENS;
    const bool ws_aligned = workspace != nullptr && aligned16(workspace);
    const size_t have = ws_aligned ? workspace_bytes : 0;
    const size_t split_bytes = pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim,
                                                          max_blocks_per_seq, partition_tokens);
    DecodePlan plan{variant, 1};
    if (variant == PKV_DECODE_AUTO)
        plan = plan_auto(num_seqs, num_heads, num_kv_heads, max_blocks_per_seq, partition_tokens,
                         have, split_bytes);
    else if (variant == PKV_DECODE_CLUSTER)
        plan.parts = cluster_parts_for(max_blocks_per_seq, partition_tokens);
    if (plan.variant == PKV_DECODE_SPLIT && have < split_bytes) return PKV_ERR_WORKSPACE;

    CUtensorMap tmk, tmv;
    if (!encode_cache_map(&tmk, k_cache, rows, head_dim) ||
        !encode_cache_map(&tmv, v_cache, rows, head_dim))
        return PKV_ERR_CUDA;

    pkv::DecodeParams p{};
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.err = err_word;
    p.num_blocks = num_blocks;
    p.W = max_blocks_per_seq;
    p.B = num_seqs;
    p.Hq = num_heads;
    p.Hkv = num_kv_heads;
    p.group = num_heads / num_kv_heads;
    p.chunks = (p.group + 7) / 8;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.k_new = static_cast<const __nv_bfloat16 *>(k_new);
    p.v_new = static_cast<const __nv_bfloat16 *>(v_new);
    p.k_cache = static_cast<__nv_bfloat16 *>(const_cast<void *>(k_cache));
    p.v_cache = static_cast<__nv_bfloat16 *>(const_cast<void *>(v_cache));
    int mode = 0;  // single pass
    bool use_order = false;
    if (plan.variant == PKV_DECODE_SPLIT) {
        mode = 1;
        p.part_blocks = part_blocks;
        p.num_parts = num_parts_for(max_blocks_per_seq, partition_tokens);
        p.ws_parts = p.num_parts;
        const size_t rows_ws = static_cast<size_t>(num_seqs) * num_heads * p.ws_parts;
        p.ws_o = static_cast<float *>(workspace);
        p.ws_ml = p.ws_o + rows_ws * head_dim;
    } else if (plan.variant == PKV_DECODE_CLUSTER) {
        mode = 2;
        p.part_blocks = 0;  // per sequence: its blocks / num_parts
        p.num_parts = plan.parts;
        // longest sequences first when there are enough of them to matter
        use_order = num_seqs >= 16 && have >= order_bytes(num_seqs);
    } else {
        p.part_blocks = max_blocks_per_seq;
        p.num_parts = 1;
        // longest sequences first, when the workspace has room for the order
        use_order = have >= static_cast<size_t>(num_seqs) * sizeof(int32_t);
    }
    if (use_order) {
        int32_t *order = static_cast<int32_t *>(workspace);
        cudaError_t e = pkv::launch_order(seq_lens, num_seqs, max_blocks_per_seq, order,
                                          static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_status(e);
        p.order = order;
    }
    pkv::DecodeTuning t{env_int("PKV_DECODE_WARPS", 4), env_int("PKV_DECODE_STAGES", 2)};
    cudaError_t e = pkv::launch_decode(tmk, tmv, p, head_dim, mode, t,
                                       static_cast<cudaStream_t>(stream));
    return cuda_status(e);
}

pkv_status pkv_paged_attention_decode_ex(void *out, const void *q, const void *k_cache,
                                         const void *v_cache, const int32_t *block_tables,
                                         int max_blocks_per_seq, const int32_t *seq_lens,
                                         int num_seqs, int num_heads, int num_kv_heads,
                                         int head_dim, int64_t num_blocks, float scale,
                                         int variant, int partition_tokens, void *workspace,
                                         size_t workspace_bytes, unsigned int *err_word,
                                         void *stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, num_blocks, scale, variant,
                       partition_tokens, workspace, workspace_bytes, err_word, stream, nullptr,
                       nullptr);
}

pkv_status pkv_paged_decode_step(void *out, const void *q, const void *k_new, const void *v_new,
                                 void *k_cache, void *v_cache, const int32_t *block_tables,
                                 int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
                                 int num_heads, int num_kv_heads, int head_dim,
                                 int64_t num_blocks, float scale, int variant,
                                 int partition_tokens, void *workspace, size_t workspace_bytes,
                                 unsigned int *err_word, void *stream) {
    if (num_seqs > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)))
        return PKV_ERR_INVALID_ARG;
    return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, num_blocks, scale, variant,
                       partition_tokens, workspace, workspace_bytes, err_word, stream, k_new,
                       v_new);
}

size_t pkv_decode_prefix_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                         int max_blocks_per_seq, int partition_tokens) {
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || max_blocks_per_seq <= 0) return 0;
    if (partition_tokens <= 0) partition_tokens = kDefaultPartitionTokens;
    if (partition_tokens % PKV_BLOCK_TOKENS) return 0;
    const size_t parts =
        static_cast<size_t>(num_parts_for(max_blocks_per_seq, partition_tokens)) +
        (max_blocks_per_seq + pkv::kPrefixSpanBlocks - 1) / pkv::kPrefixSpanBlocks;
    return static_cast<size_t>(num_seqs) * num_heads * parts * (static_cast<size_t>(head_dim) + 2) *
           sizeof(float);
}

static pkv_status prefix_impl(void *out, const void *q, const void *k_cache,
                                             const void *v_cache, const int32_t *block_tables,
                                             int max_blocks_per_seq, const int32_t *seq_lens,
                                             int num_seqs, int num_heads, int num_kv_heads,
                                             int head_dim, int64_t num_blocks, float scale,
                                             const int32_t *prefix_blocks,
                                             const int32_t *group_offsets,
                                             const int32_t *group_seqs, int num_groups,
                                             int max_suffix_blocks, int partition_tokens,
                                             void *workspace, size_t workspace_bytes,
                                             unsigned int *err_word, void *stream,
                              const void *k_new, const void *v_new) {
    if (num_seqs < 0 || num_seqs > 65535 || num_heads <= 0 || num_kv_heads <= 0 ||
        num_heads % num_kv_heads || max_blocks_per_seq <= 0 || num_blocks <= 0 ||
        !std::isfinite(scale) || num_groups < 0 || num_groups > 65535)
        return PKV_ERR_INVALID_ARG;
    if (partition_tokens <= 0) partition_tokens = kDefaultPartitionTokens;
    if (partition_tokens % PKV_BLOCK_TOKENS || partition_tokens > 65536) return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !prefix_blocks ||
        (num_groups > 0 && (!group_offsets || !group_seqs)))
        return PKV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_ERR_INVALID_ARG;
    if (num_blocks > INT32_MAX / PKV_BLOCK_TOKENS / num_kv_heads) return PKV_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(max_blocks_per_seq) * PKV_BLOCK_TOKENS > INT32_MAX)
        return PKV_ERR_INVALID_ARG;
    const size_t need = pkv_decode_prefix_workspace_bytes(num_seqs, num_heads, head_dim,
                                                          max_blocks_per_seq, partition_tokens);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return PKV_ERR_WORKSPACE;

    const int64_t rows = num_blocks * num_kv_heads * PKV_BLOCK_TOKENS;
    CUtensorMap tmk, tmv;
    if (!encode_cache_map(&tmk, k_cache, rows, head_dim) ||
        !encode_cache_map(&tmv, v_cache, rows, head_dim))
        return PKV_ERR_CUDA;

    // suffix partitions the grid covers: from the caller's bound on the blocks
    // past each prefix (no empty partitions), else from the table width
    const int suffix_blocks = max_suffix_blocks > 0 && max_suffix_blocks < max_blocks_per_seq
                                  ? max_suffix_blocks
                                  : max_blocks_per_seq;
    const int suffix_parts = num_parts_for(suffix_blocks, partition_tokens);
    const int prefix_parts = (max_blocks_per_seq + pkv::kPrefixSpanBlocks - 1) / pkv::kPrefixSpanBlocks;
    const size_t ws_rows = static_cast<size_t>(num_seqs) * num_heads * (prefix_parts + suffix_parts);
    float *ws_o = static_cast<float *>(workspace);
    float *ws_ml = ws_o + ws_rows * head_dim;

    pkv::PrefixParams pp{};
    pp.out = static_cast<__nv_bfloat16 *>(out);
    pp.q = static_cast<const __nv_bfloat16 *>(q);
    pp.block_tables = block_tables;
    pp.seq_lens = seq_lens;
    pp.prefix_blocks = prefix_blocks;
    pp.group_offsets = group_offsets;
    pp.group_seqs = group_seqs;
    pp.ws_o = ws_o;
    pp.ws_ml = ws_ml;
    pp.err = err_word;
    pp.num_blocks = num_blocks;
    pp.W = max_blocks_per_seq;
    pp.B = num_seqs;
    pp.Hq = num_heads;
    pp.Hkv = num_kv_heads;
    pp.group = num_heads / num_kv_heads;
    pp.ws_parts = prefix_parts + suffix_parts;
    pp.prefix_parts = prefix_parts;
    pp.part_blocks = partition_tokens / PKV_BLOCK_TOKENS;
    pp.scale_log2 = scale * 1.4426950408889634f;

    pkv::DecodeParams dp{};
    dp.out = pp.out;
    dp.q = pp.q;
    dp.block_tables = block_tables;
    dp.seq_lens = seq_lens;
    dp.err = err_word;
    dp.num_blocks = num_blocks;
    dp.W = max_blocks_per_seq;
    dp.B = num_seqs;
    dp.Hq = num_heads;
    dp.Hkv = num_kv_heads;
    dp.group = pp.group;
    dp.chunks = (pp.group + 7) / 8;
    dp.scale_log2 = pp.scale_log2;
    dp.part_blocks = pp.part_blocks;
    dp.num_parts = suffix_parts;
    dp.ws_o = ws_o;
    dp.ws_ml = ws_ml;
    dp.ws_parts = pp.ws_parts;
    dp.ws_part0 = prefix_parts;
    dp.start_blocks = prefix_blocks;
    dp.skip_merge = true;
    dp.k_new = static_cast<const __nv_bfloat16 *>(k_new);
    dp.v_new = static_cast<const __nv_bfloat16 *>(v_new);
    dp.k_cache = static_cast<__nv_bfloat16 *>(const_cast<void *>(k_cache));
    dp.v_cache = static_cast<__nv_bfloat16 *>(const_cast<void *>(v_cache));

    cudaError_t e = pkv::launch_cascade(tmk, tmv, pp, dp, head_dim, num_groups,
                                        static_cast<cudaStream_t>(stream));
    return cuda_status(e);
}

pkv_status pkv_paged_attention_decode_prefix(void *out, const void *q, const void *k_cache,
                                             const void *v_cache, const int32_t *block_tables,
                                             int max_blocks_per_seq, const int32_t *seq_lens,
                                             int num_seqs, int num_heads, int num_kv_heads,
                                             int head_dim, int64_t num_blocks, float scale,
                                             const int32_t *prefix_blocks,
                                             const int32_t *group_offsets,
                                             const int32_t *group_seqs, int num_groups,
                                             int max_suffix_blocks, int partition_tokens,
                                             void *workspace, size_t workspace_bytes,
                                             unsigned int *err_word, void *stream) {
    return prefix_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, num_blocks, scale,
                       prefix_blocks, group_offsets, group_seqs, num_groups, max_suffix_blocks,
                       partition_tokens, workspace, workspace_bytes, err_word, stream, nullptr,
                       nullptr);
}

pkv_status pkv_paged_decode_prefix_step(void *out, const void *q, const void *k_new,
                                        const void *v_new, void *k_cache, void *v_cache,
                                        const int32_t *block_tables, int max_blocks_per_seq,
                                        const int32_t *seq_lens, int num_seqs, int num_heads,
                                        int num_kv_heads, int head_dim, int64_t num_blocks,
                                        float scale, const int32_t *prefix_blocks,
                                        const int32_t *group_offsets, const int32_t *group_seqs,
                                        int num_groups, int max_suffix_blocks,
                                        int partition_tokens, void *workspace,
                                        size_t workspace_bytes, unsigned int *err_word,
                                        void *stream) {
    if (num_seqs > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)))
        return PKV_ERR_INVALID_ARG;
    return prefix_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, num_blocks, scale,
                       prefix_blocks, group_offsets, group_seqs, num_groups, max_suffix_blocks,
                       partition_tokens, workspace, workspace_bytes, err_word, stream, k_new,
                       v_new);
}

pkv_status pkv_paged_attention_prefill(void *out, const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       int max_blocks_per_seq, const int32_t *seq_lens,
                                       const int32_t *query_start, int num_seqs, int max_query_len,
                                       int num_heads, int num_kv_heads, int head_dim,
                                       int64_t num_blocks, float scale, unsigned int *err_word,
                                       void *stream) {
    if (num_seqs < 0 || num_seqs > 65535 || max_query_len < 0 || num_heads <= 0 ||
        num_kv_heads <= 0 || num_kv_heads > 65535 || num_heads % num_kv_heads ||
        max_blocks_per_seq <= 0 || num_blocks <= 0 || !std::isfinite(scale))
        return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0 || max_query_len == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !query_start)
        return PKV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_ERR_INVALID_ARG;
    if (num_blocks > INT32_MAX / PKV_BLOCK_TOKENS / num_kv_heads) return PKV_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(max_blocks_per_seq) * PKV_BLOCK_TOKENS > INT32_MAX)
        return PKV_ERR_INVALID_ARG;
    const int64_t rows = num_blocks * num_kv_heads * PKV_BLOCK_TOKENS;
    CUtensorMap tmk, tmv;
    if (!encode_cache_map(&tmk, k_cache, rows, head_dim) ||
        !encode_cache_map(&tmv, v_cache, rows, head_dim))
        return PKV_ERR_CUDA;
    pkv::PrefillParams p{};
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.query_start = query_start;
    p.err = err_word;
    p.num_blocks = num_blocks;
    p.W = max_blocks_per_seq;
    p.B = num_seqs;
    p.Hq = num_heads;
    p.Hkv = num_kv_heads;
    p.group = num_heads / num_kv_heads;
    p.scale_log2 = scale * 1.4426950408889634f;
    cudaError_t e = pkv::launch_prefill_tc(tmk, tmv, p, head_dim, max_query_len, sm_count(),
                                           static_cast<cudaStream_t>(stream));
    return cuda_status(e);
}

pkv_status pkv_paged_attention_decode(void *out, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *block_tables,
                                      int max_blocks_per_seq, const int32_t *seq_lens,
                                      int num_seqs, int num_heads, int num_kv_heads,
                                      int head_dim, int64_t num_blocks, float scale,
                                      void *workspace, size_t workspace_bytes,
                                      unsigned int *err_word, void *stream) {
    return pkv_paged_attention_decode_ex(out, q, k_cache, v_cache, block_tables,
                                         max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                                         num_kv_heads, head_dim, num_blocks, scale,
                                         PKV_DECODE_AUTO, kDefaultPartitionTokens, workspace,
                                         workspace_bytes, err_word, stream);
}

}  // extern "C"
