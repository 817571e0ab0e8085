// Paged decode attention for sm_100a.
//
// What is computed ("vLLM 與 PagedAttention：高吞吐推理的關鍵", section 三, step
// 三: attention over all earlier K/V looked up through the block table; section
// 二: 16-token blocks, logical block i -> physical block table[i]):
//   out[b][h] = softmax_p(scale * q[b][h] . K_b[p]) V_b[p],   p in [0, len_b)
// with query head h reading KV head h / (Hq / Hkv).
//
// Work unit: one CTA per (sequence, KV head [, chunk of <= 8 query heads],
// partition).  The single-pass variant makes the partition the whole table
// row; split-K cuts it into fixed token partitions whose partial results
// (running max m, sum l, unnormalised o, all fp32, log2 domain) a second
// kernel merges by log-sum-exp.
//
// Inside a CTA, NW consumer warps take the unit's logical blocks round-robin.
// Each warp runs its own S-stage ring: its lane 0 issues TMA tile loads of
// the K and V tiles of one (physical block, KV head) -- 16 rows x head_dim
// bf16, each a contiguous 2-4 KB range of the cache -- into 128-byte-swizzled
// shared memory, with completion counted on a per-stage mbarrier.  The block
// table row is read ahead into registers, 32 entries per lane-load, so the
// dependent table -> TMA chain never waits on a table read.  Waits are
// bounded (PKV_DEV_ERR_TIMEOUT) and every issued copy is drained before exit.
//
// Inner products:
//  * Hq == Hkv (one query row per KV head): CUDA cores.  Lane (c, g) owns
//    16-byte column chunk c of rows g, g+RG, ...; partial dot products are
//    combined by a butterfly reduce-scatter (log2(16/RG)+1 shuffles for 16
//    rows instead of 4 per row), fp32 online softmax in the exp2 domain, and
//    P.V accumulated in fp32 per owned chunk.
//  * grouped heads (Hq > Hkv): the group makes a real dense tile, so tensor
//    cores take it.  S^T[16 tokens x 8 heads] = K_tile . Q^T with mma.m16n8k16
//    (tokens on M, the query group padded to N = 8), the softmax runs on the
//    accumulator fragments, P is moved into the B-operand layout with
//    movmatrix, and O^T[d x 8] += V^T . P^T with V^T read by ldmatrix.trans.
//    K and V stay bf16 (as stored), products accumulate in fp32.
#include "decode_unit.cuh"

namespace pkv {

namespace {

using namespace dev;

template <int D, int NW, int S, bool MMA, int MODE>
__global__ void __launch_bounds__(NW * 32)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const DecodeParams p) {
    // The preceding grid (the order kernel, or the previous call's last grid):
    // with an order it is read first; otherwise the unit reads the sequence's
    // length and table row before waiting for that grid, so that a step's
    // grid, resident while the previous one drains, starts its K/V loads as
    // soon as it is released.
    if (p.order != nullptr) {
        pdl_wait_primary();
        decode_unit<D, NW, S, MMA, MODE>(tmk, tmv, p, blockIdx.x, blockIdx.y, __ldg(p.order + blockIdx.z));
    } else {
        decode_unit<D, NW, S, MMA, MODE>(tmk, tmv, p, blockIdx.x, blockIdx.y, static_cast<int>(blockIdx.z),
                                         true);
    }
}

// Longest-first order of the sequences by block count (counting sort; ties in
// any order -- the order only steers scheduling, never the arithmetic).
constexpr int kOrderThreads = 1024;
constexpr int kOrderBuckets = 4096;

__global__ void __launch_bounds__(kOrderThreads)
    order_kernel(const int32_t *__restrict__ seq_lens, int B, int W, int shift, int32_t *order) {
    pdl_launch_dependents();
    // the counting and the scan read only the lengths: they run before the
    // wait for the previous call's grid, which still reads the old order
    __shared__ int count[kOrderBuckets];
    __shared__ int warp_tot[kOrderThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < kOrderBuckets; i += kOrderThreads) count[i] = 0;
    __syncthreads();
    const auto bucket = [&](int b) {  // descending: the longest sequences get bucket 0
        int len = __ldg(seq_lens + b);
        len = len < 0 ? 0 : min(len, W * kBlockTokens);
        const int nblk = (len + kBlockTokens - 1) / kBlockTokens;
        return (kOrderBuckets - 1) - min(nblk >> shift, kOrderBuckets - 1);
    };
    for (int b = tid; b < B; b += kOrderThreads) atomicAdd(&count[bucket(b)], 1);
    __syncthreads();
    // exclusive scan of the bucket counts: each thread owns 4 consecutive buckets
    constexpr int kPer = kOrderBuckets / kOrderThreads;
    int local[kPer], sum = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        local[i] = count[tid * kPer + i];
        sum += local[i];
    }
    int incl = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    int run = before + incl - sum;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        count[tid * kPer + i] = run;  // now the next free position of the bucket
        run += local[i];
    }
    __syncthreads();
    pdl_wait_primary();
    for (int b = tid; b < B; b += kOrderThreads) order[atomicAdd(&count[bucket(b)], 1)] = b;
}

// Log-sum-exp merge of the split-K partitions of one (sequence, query head):
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.
// The (m, l) pairs of all partitions are read at once into shared memory and
// their weights computed once; each thread then sums its output column over
// the partitions with the loads batched.  Partitions are combined in index
// order, so the result does not depend on which CTA finished first.
template <int D>
__global__ void __launch_bounds__(D) splitk_merge_kernel(const DecodeParams p) {
    constexpr int kMaxParts = 256;  // per pass; longer rows loop
    constexpr int kFewParts = 16;   // rows with at most this many partials: all loads at once
    __shared__ float s_w[kMaxParts];
    __shared__ float s_red[D / 32][2];
    pdl_launch_dependents();  // the next call's first grid may be scheduled
    const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
    // the partition count comes from the decode's inputs, read before the wait
    int len = __ldg(p.seq_lens + b);
    len = len < 0 ? 0 : min(len, p.W * kBlockTokens);
    int start = 0;
    if (p.start_blocks != nullptr) start = min(max(__ldg(p.start_blocks + b), 0), len / kBlockTokens);
    const int nblk = (len + kBlockTokens - 1) / kBlockTokens;
    const int np = (nblk - start + p.part_blocks - 1) / p.part_blocks;
    const size_t row = static_cast<size_t>(b) * p.Hq + h;
    const float *ml = p.ws_ml + 2 * (row * p.ws_parts + p.ws_part0);
    const float *o = p.ws_o + (row * p.ws_parts + p.ws_part0) * D;
    pdl_wait_primary();  // the decode grid's partials
    if (np <= kFewParts) {
        float mv[kFewParts], lv[kFewParts], ov[kFewParts];
#pragma unroll
        for (int q = 0; q < kFewParts; ++q) {
            mv[q] = -INFINITY;
            lv[q] = 0.f;
            ov[q] = 0.f;
            if (q < np) {
                const float2 v = *reinterpret_cast<const float2 *>(ml + 2 * q);
                mv[q] = v.x;
                lv[q] = v.y;
                ov[q] = o[static_cast<size_t>(q) * D + e];
            }
        }
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < kFewParts; ++q) M = fmaxf(M, mv[q]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int q = 0; q < kFewParts; ++q) {
                const float w = mv[q] == -INFINITY ? 0.f : exp2f(mv[q] - M);
                L = fmaf(lv[q], w, L);
                O = fmaf(ov[q], w, O);
            }
        }
        p.out[row * D + e] = __float2bfloat16(L > 0.f ? O / L : 0.f);
        return;
    }
    // M over all partitions
    float mx = -INFINITY;
    for (int q = e; q < np; q += D) mx = fmaxf(mx, ml[2 * q]);
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    if ((e & 31) == 0) s_red[e >> 5][0] = mx;
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) M = fmaxf(M, s_red[w][0]);
    float L = 0.f, O = 0.f;
    for (int base = 0; base < np; base += kMaxParts) {
        const int n = min(kMaxParts, np - base);
        __syncthreads();  // s_w and s_red reuse
        float lsum = 0.f;
        for (int q = e; q < n; q += D) {
            const float2 v = *reinterpret_cast<const float2 *>(ml + 2 * (base + q));
            const float w = v.x == -INFINITY ? 0.f : exp2f(v.x - M);
            s_w[q] = w;
            lsum = fmaf(v.y, w, lsum);
        }
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, m);
        if ((e & 31) == 0) s_red[e >> 5][1] = lsum;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < D / 32; ++w) L += s_red[w][1];
        const float *ob = o + static_cast<size_t>(base) * D + e;
        int q = 0;
        for (; q + 8 <= n; q += 8) {
            float x[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = ob[static_cast<size_t>(q + i) * D];
#pragma unroll
            for (int i = 0; i < 8; ++i) O = fmaf(x[i], s_w[q + i], O);
        }
        for (; q < n; ++q) O = fmaf(ob[static_cast<size_t>(q) * D], s_w[q], O);
    }
    p.out[row * D + e] = __float2bfloat16(L > 0.f ? O / L : 0.f);
}

template <int D, int NW, int S, bool MMA, int MODE>
cudaError_t launch_one(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                       cudaStream_t stream) {
    using G = Geometry<D, NW, S>;
    constexpr int kSmem = G::kSmemBytes + (MODE == kModeCluster ? cluster_land_bytes<D, MMA>() : 0);
    auto kern = paged_decode_kernel<D, NW, S, MMA, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(p.num_parts),
                    static_cast<unsigned>(MMA ? p.Hkv * p.chunks : p.Hq),
                    static_cast<unsigned>(p.B));
    {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(NW * 32);
        cfg.dynamicSmemBytes = kSmem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        unsigned n = 0;
        // a programmatic dependent of the preceding grid (the order kernel, or
        // the previous call's last grid): it waits before it reads anything
        // that grid may write
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n++].val.programmaticStreamSerializationAllowed = 1;
        if (MODE == kModeCluster) {  // the parts of one (sequence, head) form a cluster
            attr[n].id = cudaLaunchAttributeClusterDimension;
            attr[n].val.clusterDim.x = static_cast<unsigned>(p.num_parts);
            attr[n].val.clusterDim.y = 1;
            attr[n++].val.clusterDim.z = 1;
        }
        cfg.attrs = attr;
        cfg.numAttrs = n;
        e = cudaLaunchKernelEx(&cfg, kern, tmk, tmv, p);
    }
    if (e != cudaSuccess || MODE != kModeSplit || p.skip_merge) return e;
    return launch_dependent(splitk_merge_kernel<D>, dim3(static_cast<unsigned>(p.Hq), static_cast<unsigned>(p.B)),
                            dim3(D), stream, p);
}

template <int D, bool MMA, int MODE>
cudaError_t launch_tuned(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                         DecodeTuning t, cudaStream_t stream) {
    // 4 warps x 2 stages (64 KB of ring at d = 128, three CTAs per SM) measured
    // fastest on every workload (against 1, 2 and 8 warps and 3-4 stages); the
    // other shapes stay for tuning sweeps.
    if (t.warps == 4 && t.stages == 3) return launch_one<D, 4, 3, MMA, MODE>(tmk, tmv, p, stream);
    if (t.warps == 2 && t.stages == 2) return launch_one<D, 2, 2, MMA, MODE>(tmk, tmv, p, stream);
    return launch_one<D, 4, 2, MMA, MODE>(tmk, tmv, p, stream);
}

template <int D, bool MMA>
cudaError_t launch_m(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                     int mode, DecodeTuning t, cudaStream_t stream) {
    if (mode == kModeSplit) return launch_tuned<D, MMA, kModeSplit>(tmk, tmv, p, t, stream);
    // cluster mode: 4 x 2 only (part 0's ring holds the other parts' rows of a head group)
    if (mode == kModeCluster) return launch_one<D, 4, 2, MMA, kModeCluster>(tmk, tmv, p, stream);
    return launch_tuned<D, MMA, kModeSingle>(tmk, tmv, p, t, stream);
}

template <int D>
cudaError_t launch_d(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                     int mode, DecodeTuning t, cudaStream_t stream) {
    return p.group > 1 ? launch_m<D, true>(tmk, tmv, p, mode, t, stream)
                       : launch_m<D, false>(tmk, tmv, p, mode, t, stream);
}

}  // namespace

cudaError_t launch_order(const int32_t *seq_lens, int B, int W, int32_t *order, cudaStream_t stream) {
    int shift = 0;
    while ((W >> shift) >= kOrderBuckets) ++shift;
    return launch_dependent(order_kernel, dim3(1), dim3(kOrderThreads), stream, seq_lens, B, W, shift,
                            order);
}

cudaError_t launch_decode(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                          int head_dim, int mode, DecodeTuning tuning, cudaStream_t stream) {
    if (mode != dev::kModeSingle && mode != dev::kModeSplit && mode != dev::kModeCluster)
        return cudaErrorInvalidValue;
    if (mode == dev::kModeCluster && (p.num_parts < 1 || p.num_parts > kMaxClusterParts))
        return cudaErrorInvalidValue;
    if (head_dim == 128) return launch_d<128>(tmk, tmv, p, mode, tuning, stream);
    if (head_dim == 64) return launch_d<64>(tmk, tmv, p, mode, tuning, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pkv
