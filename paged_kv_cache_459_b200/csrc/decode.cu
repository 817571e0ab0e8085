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

template <int D, int NW, int S, bool MMA, bool SPLIT>
__global__ void __launch_bounds__(NW * 32)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const DecodeParams p) {
    decode_unit<D, NW, S, MMA, SPLIT>(tmk, tmv, p, blockIdx.x, blockIdx.y, blockIdx.z);
}

// Log-sum-exp merge of the split-K partitions of one (sequence, query head):
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.
// Partitions are visited in index order, so the result does not depend on
// which CTA finished first.
template <int D>
__global__ void __launch_bounds__(D) splitk_merge_kernel(const DecodeParams p) {
    const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
    int len = __ldg(p.seq_lens + b);
    len = len < 0 ? 0 : min(len, p.W * kBlockTokens);
    const int part_tokens = p.part_blocks * kBlockTokens;
    const int np = (len + part_tokens - 1) / part_tokens;
    const size_t row = static_cast<size_t>(b) * p.Hq + h;
    const float *ml = p.ws_ml + 2 * (row * p.ws_parts + p.ws_part0);
    const float *o = p.ws_o + (row * p.ws_parts + p.ws_part0) * D;
    float M = -INFINITY;
    for (int q = 0; q < np; ++q) M = fmaxf(M, ml[2 * q]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
        for (int q = 0; q < np; ++q) {
            const float c = exp2f(ml[2 * q] - M);
            L = fmaf(ml[2 * q + 1], c, L);
            O = fmaf(o[static_cast<size_t>(q) * D + e], c, O);
        }
    }
    p.out[row * D + e] = __float2bfloat16(L > 0.f ? O / L : 0.f);
}

template <int D, int NW, int S, bool MMA, bool SPLIT>
cudaError_t launch_one(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                       cudaStream_t stream) {
    using G = Geometry<D, NW, S>;
    auto kern = paged_decode_kernel<D, NW, S, MMA, SPLIT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         G::kSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(p.num_parts),
                    static_cast<unsigned>(MMA ? p.Hkv * p.chunks : p.Hq),
                    static_cast<unsigned>(p.B));
    kern<<<grid, NW * 32, G::kSmemBytes, stream>>>(tmk, tmv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess || !SPLIT || p.skip_merge) return e;
    splitk_merge_kernel<D><<<dim3(static_cast<unsigned>(p.Hq), static_cast<unsigned>(p.B)), D, 0,
                             stream>>>(p);
    return cudaGetLastError();
}

template <int D, bool MMA, bool SPLIT>
cudaError_t launch_tuned(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                         DecodeTuning t, cudaStream_t stream) {
    // 4 warps x 2 stages (64 KB of ring at d = 128, three CTAs per SM) measured
    // fastest on every workload (against 1, 2 and 8 warps and 3-4 stages); the
    // other shapes stay for tuning sweeps.
    if (t.warps == 4 && t.stages == 3) return launch_one<D, 4, 3, MMA, SPLIT>(tmk, tmv, p, stream);
    if (t.warps == 2 && t.stages == 2) return launch_one<D, 2, 2, MMA, SPLIT>(tmk, tmv, p, stream);
    return launch_one<D, 4, 2, MMA, SPLIT>(tmk, tmv, p, stream);
}

template <int D>
cudaError_t launch_d(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                     bool split, DecodeTuning t, cudaStream_t stream) {
    const bool mma = p.group > 1;
    if (mma)
        return split ? launch_tuned<D, true, true>(tmk, tmv, p, t, stream)
                     : launch_tuned<D, true, false>(tmk, tmv, p, t, stream);
    return split ? launch_tuned<D, false, true>(tmk, tmv, p, t, stream)
                 : launch_tuned<D, false, false>(tmk, tmv, p, t, stream);
}

}  // namespace

cudaError_t launch_decode(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeParams &p,
                          int head_dim, bool split, DecodeTuning tuning, cudaStream_t stream) {
    if (head_dim == 128) return launch_d<128>(tmk, tmv, p, split, tuning, stream);
    if (head_dim == 64) return launch_d<64>(tmk, tmv, p, split, tuning, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pkv
