// Paged KV-cache write: scatter each new token's K and V rows into the slot
// the block manager handed out ("vLLM 與 PagedAttention：高吞吐推理的關鍵",
// section 三, step 三: write into the current block, or a new one when full).
//
// One thread per 16-byte vector of a (token, KV head) row; K and V move in
// the same thread.  A few MB per decode step at most, so the kernel is
// launch- and latency-bound; coalesced 16-byte loads and stores are all it
// needs.  Bit-exact: plain copies, no arithmetic on the values.
#include <algorithm>

#include "../../include/pkv.h"
#include "internal.h"

namespace pkv {

__global__ void __launch_bounds__(256) kv_write_kernel(const uint4 *__restrict__ k,
                                                       const uint4 *__restrict__ v,
                                                       uint4 *__restrict__ k_cache,
                                                       uint4 *__restrict__ v_cache,
                                                       const int64_t *__restrict__ slots,
                                                       long long total, int vec_per_row, int Hkv,
                                                       long long num_blocks, unsigned int *err) {
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int vec = static_cast<int>(idx % vec_per_row);
    const long long row = idx / vec_per_row;
    const int h = static_cast<int>(row % Hkv);
    const long long t = row / Hkv;
    const long long slot = slots[t];
    if (slot < 0) return;
    if (slot >= num_blocks * kBlockTokens) {
        if (err != nullptr && vec == 0 && h == 0) atomicOr(err, PKV_DEV_ERR_BAD_SLOT);
        return;
    }
    const long long blk = slot / kBlockTokens;
    const int off = static_cast<int>(slot % kBlockTokens);
    const long long dst = ((blk * Hkv + h) * kBlockTokens + off) * vec_per_row + vec;
    const uint4 kv = __ldg(k + idx);
    const uint4 vv = __ldg(v + idx);
    k_cache[dst] = kv;
    v_cache[dst] = vv;
}

cudaError_t launch_kv_write(const void *k, const void *v, void *k_cache, void *v_cache,
                            const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                            int head_dim, long long num_blocks, unsigned int *err,
                            cudaStream_t stream) {
    const int vec_per_row = head_dim / 8;
    const long long total = static_cast<long long>(num_tokens) * num_kv_heads * vec_per_row;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const long long blocks = (total + threads - 1) / threads;
    kv_write_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<uint4 *>(k_cache),
        static_cast<uint4 *>(v_cache), slot_mapping, total, vec_per_row, num_kv_heads, num_blocks,
        err);
    return cudaGetLastError();
}

// Whole-block copies (copy-on-write): pair blockIdx.y, 16-byte vectors over
// the block's Hkv x 16 x d elements of both caches.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4 *__restrict__ k_cache,
                                                          uint4 *__restrict__ v_cache,
                                                          const int64_t *__restrict__ src,
                                                          const int64_t *__restrict__ dst,
                                                          long long vec_per_block,
                                                          long long num_blocks, unsigned int *err) {
    const long long s = src[blockIdx.y], d = dst[blockIdx.y];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) {
        if (err != nullptr && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(err, PKV_DEV_ERR_BAD_BLOCK);
        return;
    }
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < vec_per_block;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        k_cache[d * vec_per_block + i] = k_cache[s * vec_per_block + i];
        v_cache[d * vec_per_block + i] = v_cache[s * vec_per_block + i];
    }
}

cudaError_t launch_copy_blocks(void *k_cache, void *v_cache, const int64_t *src, const int64_t *dst,
                               int n, int num_kv_heads, int head_dim, long long num_blocks,
                               unsigned int *err, cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const long long vec = static_cast<long long>(num_kv_heads) * kBlockTokens * head_dim / 8;
    const long long per_cta = 256 * 4;
    const unsigned gx = static_cast<unsigned>(std::min<long long>((vec + per_cta - 1) / per_cta, 1024));
    copy_blocks_kernel<<<dim3(gx, static_cast<unsigned>(n)), 256, 0, stream>>>(
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), src, dst, vec, num_blocks, err);
    return cudaGetLastError();
}

// Block swap over the host link: pair blockIdx.y; the host side is pinned,
// device-mapped memory reached directly by the loads or stores.
__global__ void __launch_bounds__(256) swap_blocks_kernel(uint4 *k_cache, uint4 *v_cache,
                                                          uint4 *host_k, uint4 *host_v,
                                                          const int64_t *__restrict__ gpu_blocks,
                                                          const int64_t *__restrict__ host_blocks,
                                                          int direction, long long vec_per_block,
                                                          long long num_blocks,
                                                          long long num_host_blocks,
                                                          unsigned int *err) {
    const long long g = gpu_blocks[blockIdx.y], h = host_blocks[blockIdx.y];
    if (g < 0 || g >= num_blocks || h < 0 || h >= num_host_blocks) {
        if (err != nullptr && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(err, PKV_DEV_ERR_BAD_BLOCK);
        return;
    }
    uint4 *dk = direction == PKV_SWAP_OUT ? host_k + h * vec_per_block : k_cache + g * vec_per_block;
    uint4 *dv = direction == PKV_SWAP_OUT ? host_v + h * vec_per_block : v_cache + g * vec_per_block;
    const uint4 *sk = direction == PKV_SWAP_OUT ? k_cache + g * vec_per_block : host_k + h * vec_per_block;
    const uint4 *sv = direction == PKV_SWAP_OUT ? v_cache + g * vec_per_block : host_v + h * vec_per_block;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < vec_per_block;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        dk[i] = sk[i];
        dv[i] = sv[i];
    }
}

cudaError_t launch_swap_blocks(void *k_cache, void *v_cache, void *host_k, void *host_v,
                               const int64_t *gpu_blocks, const int64_t *host_blocks, int n,
                               int direction, int num_kv_heads, int head_dim, long long num_blocks,
                               long long num_host_blocks, unsigned int *err, cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const long long vec = static_cast<long long>(num_kv_heads) * kBlockTokens * head_dim / 8;
    const unsigned gx = static_cast<unsigned>(std::min<long long>((vec + 1023) / 1024, 256));
    swap_blocks_kernel<<<dim3(gx, static_cast<unsigned>(n)), 256, 0, stream>>>(
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), static_cast<uint4 *>(host_k),
        static_cast<uint4 *>(host_v), gpu_blocks, host_blocks, direction, vec, num_blocks,
        num_host_blocks, err);
    return cudaGetLastError();
}

}  // namespace pkv
