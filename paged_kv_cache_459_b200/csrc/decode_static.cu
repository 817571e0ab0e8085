// Split-K decode attention whose scratch lives in a fixed device array of
// this library, so the call allocates nothing.
//
// Who needs it: callers that may not allocate device memory at the point
// where they run decode -- an inference-engine plugin whose enqueue path is
// forbidden to allocate, a serving loop that reserves all of its memory up
// front and treats any later allocation as a failure, or code running where
// cudaMalloc/cudaFree are off limits because they can synchronise the device
// or take a process-wide allocator lock.  Such callers cannot hand the
// regular entry point the workspace its split-K partials need.
//
// The scratch array below is part of the library image: every GPU that loads
// the library holds its PKV_STATIC_SCRATCH_BYTES until the process exits.
// Host code cannot use the array's name as a device address (on the host it
// names a stand-in object), so the device address is looked up once per
// device with cudaGetSymbolAddress while that device is current, and that
// address is what the kernels receive.
#include <mutex>

#include "../../include/pkv.h"
#include "internal.h"

namespace {

constexpr int kMaxDevices = 64;

// Split-K partial results (per partition: unnormalised output, max, sum).
// Nothing in it has to start at zero: the decode kernel writes every
// partition that holds tokens before the merge kernel reads it, and the merge
// reads no other partition.
__device__ __align__(256) unsigned char pkv_static_scratch[PKV_STATIC_SCRATCH_BYTES];

// The array's device address on each device, set only by a successful
// lookup: a failed one (e.g. an error left behind by an unrelated earlier
// launch) is retried by the next call instead of disabling the entry point.
struct ScratchSlot {
    std::mutex lock;
    void *addr = nullptr;
};
ScratchSlot g_slots[kMaxDevices];

// Device address of the scratch array on the current device; the first
// successful call on a device does the lookup.
cudaError_t scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    ScratchSlot &s = g_slots[dev];
    std::lock_guard<std::mutex> guard(s.lock);
    if (s.addr == nullptr) {
        void *addr = nullptr;
        e = cudaGetSymbolAddress(&addr, pkv_static_scratch);
        if (e != cudaSuccess) return e;
        if (addr == nullptr) return cudaErrorInvalidSymbol;
        s.addr = addr;
    }
    *out = s.addr;
    return cudaSuccess;
}

}  // namespace

extern "C" {

pkv_status pkv_paged_attention_decode_static(void *out, const void *q, const void *k_cache,
                                             const void *v_cache, const int32_t *block_tables,
                                             int max_blocks_per_seq, const int32_t *seq_lens,
                                             int num_seqs, int num_heads, int num_kv_heads,
                                             int head_dim, int64_t num_blocks, float scale,
                                             int partition_tokens, unsigned int *err_word,
                                             void *stream) {
    if (partition_tokens <= 0) partition_tokens = 512;
    if (num_seqs == 0) return PKV_OK;
    const size_t need = pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim,
                                                   max_blocks_per_seq, partition_tokens);
    if (need == 0) return PKV_ERR_INVALID_ARG;
    if (need > static_cast<size_t>(PKV_STATIC_SCRATCH_BYTES)) return PKV_ERR_WORKSPACE;
    void *scratch = nullptr;
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) return static_cast<pkv_status>(pkv::cuda_status(e));
    return pkv_paged_attention_decode_ex(out, q, k_cache, v_cache, block_tables,
                                         max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                                         num_kv_heads, head_dim, num_blocks, scale,
                                         PKV_DECODE_SPLIT, partition_tokens, scratch,
                                         static_cast<size_t>(PKV_STATIC_SCRATCH_BYTES), err_word,
                                         stream);
}

}  // extern "C"
