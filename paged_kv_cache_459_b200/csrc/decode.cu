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
#include "decode_common.cuh"

namespace pkv {

namespace {

using namespace dev;

// ----------------------------------------------------------------------------
template <int D, int NW, int S, bool MMA, bool SPLIT>
__global__ void __launch_bounds__(NW * 32)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const DecodeParams p) {
    using G = Geometry<D, NW, S>;
    const int part = blockIdx.x;
    const int b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kvh = MMA ? static_cast<int>(blockIdx.y) / p.chunks : static_cast<int>(blockIdx.y);
    const int chunk = MMA ? static_cast<int>(blockIdx.y) % p.chunks : 0;
    const int h0 = MMA ? kvh * p.group + chunk * 8 : kvh;  // first query head of this CTA
    const int heads = MMA ? min(8, p.group - chunk * 8) : 1;

    int len = __ldg(p.seq_lens + b);
    if (len < 0 || len > p.W * kBlockTokens) {
        if (threadIdx.x == 0 && part == 0 && blockIdx.y == 0) flag(p.err, PKV_DEV_ERR_BAD_LEN);
        len = len < 0 ? 0 : p.W * kBlockTokens;
    }
    const int nblk = (len + kBlockTokens - 1) / kBlockTokens;
    int start = 0;
    if (p.start_blocks != nullptr) start = min(max(__ldg(p.start_blocks + b), 0), len / kBlockTokens);
    const int blk_begin = max(part * p.part_blocks, start);
    const int blk_end = min(nblk, (part + 1) * p.part_blocks);
    if (blk_begin >= blk_end) {
        // Nothing to read.  Single pass: the (empty) sequence's rows are zero.
        // Split-K: the merge kernel only reads partitions that hold tokens.
        if (!SPLIT)
            for (int i = threadIdx.x; i < heads * D; i += NW * 32)
                p.out[(static_cast<size_t>(b) * p.Hq + h0 + i / D) * D + i % D] = __float2bfloat16(0.f);
        return;
    }

    extern __shared__ uint8_t smem_raw[];
    // Stage buffers must sit on 1024-byte boundaries for the 128-byte swizzle.
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = smem + warp * S * G::kStageBytes;
    const uint32_t bars = smem_u32(smem + G::kRingBytes) + warp * S * 8;

    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bars + 8 * s, 1);
        fence_mbar_init();
    }
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    __syncthreads();

    const int n_mine = blk_end - blk_begin > warp ? (blk_end - blk_begin - warp + NW - 1) / NW : 0;
    TableWindow tw;
    tw.row = p.block_tables + static_cast<size_t>(b) * p.W;
    tw.first = blk_begin + warp;
    tw.stride = NW;
    tw.count = n_mine;
    tw.init(lane);
    const uint64_t policy = l2_policy_evict_first();
    const int y_head = kvh * kBlockTokens;

    auto issue = [&](int i) {  // warp-uniform
        const int32_t phys = tw.get(i);
        if (lane == 0) {
            const uint32_t bar = bars + 8 * (i % S);
            if (phys >= 0 && phys < p.num_blocks) {
                const uint32_t dst = smem_u32(ring + (i % S) * G::kStageBytes);
                const int y = phys * (p.Hkv * kBlockTokens) + y_head;
                mbar_arrive_expect_tx(bar, G::kStageBytes);
#pragma unroll
                for (int hh = 0; hh < G::kHalves; ++hh) {
                    tma_load_2d(dst + hh * kBoxBytes, &tmk, hh * 64, y, bar, policy);
                    tma_load_2d(dst + G::kTileBytes + hh * kBoxBytes, &tmv, hh * 64, y, bar, policy);
                }
            } else {
                flag(p.err, PKV_DEV_ERR_BAD_BLOCK);
                mbar_arrive(bar);  // an empty phase: the consumer skips the block
            }
        }
    };

    using Head = typename std::conditional<MMA, GroupHeads<D>, ScalarHead<D>>::type;
    Head st;
    if constexpr (MMA)
        st.init(p.q + (static_cast<size_t>(b) * p.Hq + h0) * D, heads, p.scale_log2, lane);
    else
        st.init(p.q + (static_cast<size_t>(b) * p.Hq + h0) * D, p.scale_log2, lane);

    for (int i = 0; i < S && i < n_mine; ++i) issue(i);

    int i = 0;
    for (; i < n_mine; ++i) {
        tw.advance_to(i, lane);
        const int s = i % S;
        if (!mbar_wait(bars + 8 * s, static_cast<uint32_t>((i / S) & 1), kWaitLimitNs)) {
            if (lane == 0) flag(p.err, PKV_DEV_ERR_TIMEOUT);
            break;
        }
        const int32_t phys = tw.get(i);
        if (phys >= 0 && phys < p.num_blocks) {
            const int lb = blk_begin + warp + NW * i;
            const int nvalid = min(kBlockTokens, len - lb * kBlockTokens);
            const uint8_t *kt = ring + s * G::kStageBytes;
            if constexpr (MMA)
                st.tile(smem_u32(kt), smem_u32(kt + G::kTileBytes), nvalid, lane);
            else
                st.tile(kt, kt + G::kTileBytes, nvalid, lane);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (i + S < n_mine) issue(i + S);
    }
    if (i < n_mine) {
        // A wait gave up: let the copies still in flight land before the
        // shared memory is reused or released (again bounded).
        for (int j = i; j < n_mine && j < i + S; ++j)
            mbar_wait(bars + 8 * (j % S), static_cast<uint32_t>((j / S) & 1), kWaitLimitNs);
    }

    // ---- combine the warps of this CTA (all rings are drained) ----
    __syncthreads();
    constexpr int kRed = MMA ? 16 + 8 * D : D + 2;
    float *red = reinterpret_cast<float *>(smem);
    st.finish(red + warp * kRed, lane);
    __syncthreads();
    for (int idx = threadIdx.x; idx < heads * D; idx += NW * 32) {
        const int n = idx / D, e = idx % D;
        float mw[NW];
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            mw[w] = MMA ? red[w * kRed + n] : red[w * kRed + D];
            M = fmaxf(M, mw[w]);
        }
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float c = exp2f(mw[w] - M);
                L = fmaf(MMA ? red[w * kRed + 8 + n] : red[w * kRed + D + 1], c, L);
                O = fmaf(MMA ? red[w * kRed + 16 + n * D + e] : red[w * kRed + e], c, O);
            }
        }
        const size_t row = static_cast<size_t>(b) * p.Hq + h0 + n;
        if constexpr (SPLIT) {
            const size_t pr = row * p.ws_parts + p.ws_part0 + part;
            p.ws_o[pr * D + e] = O;
            if (e == 0) {
                p.ws_ml[2 * pr] = M;
                p.ws_ml[2 * pr + 1] = L;
            }
        } else {
            p.out[row * D + e] = __float2bfloat16(L > 0.f ? O / L : 0.f);
        }
    }
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
    // fastest on every workload; the others stay for tuning sweeps.
    if (t.warps == 4 && t.stages == 3) return launch_one<D, 4, 3, MMA, SPLIT>(tmk, tmv, p, stream);
    if (t.warps == 8 && t.stages == 2) return launch_one<D, 8, 2, MMA, SPLIT>(tmk, tmv, p, stream);
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
