// The per-unit decode kernel body (single pass and split-K), shared by the
// plain decode launch and the shared-prefix launch that runs it beside the
// prefix kernel.  Method, layouts and tiling: see decode.cu.
#pragma once

#include "decode_common.cuh"

namespace pkv {
namespace dev {

// How a decode unit's result leaves the CTA.
constexpr int kModeSingle = 0;   // the whole sequence: normalised row to `out`
constexpr int kModeSplit = 1;    // one token partition: (m, l, o) partial to the workspace
constexpr int kModeCluster = 2;  // one of p.num_parts equal parts of the sequence, the parts
                                 // a thread-block cluster, merged through its shared memory

// One work unit (partition `part` of sequence b, KV head / head chunk `by`)
// of the per-unit decode kernel, run by a CTA of NW warps.  The warps take
// the unit's blocks round-robin and are combined in shared memory at the end.
template <int D, int NW, int S, bool MMA, int MODE>
__device__ __forceinline__ void decode_unit(const CUtensorMap &tmk, const CUtensorMap &tmv,
                                            const DecodeParams &p, int part, int by, int b) {
    using G = Geometry<D, NW, S>;
    constexpr bool SPLIT = MODE == kModeSplit;
    constexpr bool CLUSTER = MODE == kModeCluster;
    // The next grid (the merge kernel, or the next call's) may be scheduled
    // as soon as every unit has started; it waits for this grid to finish.
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kvh = MMA ? by / p.chunks : by;
    const int chunk = MMA ? by % p.chunks : 0;
    const int h0 = MMA ? kvh * p.group + chunk * 8 : kvh;  // first query head of this CTA
    const int heads = MMA ? min(8, p.group - chunk * 8) : 1;

    // Round-robin: warp w takes blocks blk_begin + w, + NW, ...
    constexpr int kStride = NW;
    const int lead = warp;
    // Block-table entries of this warp's blocks, 32 per lane-load.  Where the
    // unit's first block does not depend on the length (no skipped prefix, not
    // cluster mode), they are loaded now, beside the length, for every block
    // the table row holds in this unit's range; entries past the sequence are
    // read but never used.  Otherwise after the length, below.
    const bool early_table = !CLUSTER && p.start_blocks == nullptr;
    TableWindow tw;
    tw.row = p.block_tables + static_cast<size_t>(b) * p.W;
    tw.stride = kStride;
    if (early_table) {
        const int first_blk = part * p.part_blocks;
        const int last_blk = min(p.W, first_blk + p.part_blocks);  // exclusive, within the row
        tw.first = first_blk + lead;
        tw.count = last_blk - tw.first > 0 ? (last_blk - tw.first + kStride - 1) / kStride : 0;
        tw.init(lane);
    }
    extern __shared__ uint8_t smem_raw[];
    // Stage buffers must sit on 1024-byte boundaries for the 128-byte swizzle.
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    int len = __ldg(p.seq_lens + b);
    if (len < 0 || len > p.W * kBlockTokens) {
        if (threadIdx.x == 0 && part == 0 && by == 0) flag(p.err, PKV_DEV_ERR_BAD_LEN);
        len = len < 0 ? 0 : p.W * kBlockTokens;
    }
    const int nblk = (len + kBlockTokens - 1) / kBlockTokens;
    int start = 0;
    if (p.start_blocks != nullptr) start = min(max(__ldg(p.start_blocks + b), 0), len / kBlockTokens);
    // Partitions are counted from the start block.  Cluster mode: the
    // sequence's blocks are cut into p.num_parts equal parts, one per CTA.
    const int pblk = CLUSTER ? (nblk - start + p.num_parts - 1) / p.num_parts : p.part_blocks;
    const int blk_begin = min(nblk, start + part * pblk);
    const int blk_end = min(nblk, blk_begin + pblk);
    // Cluster mode: an empty part still takes part in the merge (every CTA of
    // the cluster must reach its barriers); it contributes nothing.
    if (blk_begin >= blk_end && !CLUSTER) {
        // Nothing to read.  Single pass: the (empty) sequence's rows are zero.
        // Split-K: the merge kernel only reads partitions that hold tokens.
        // A fused write whose token lies before the start block (inside a
        // shared prefix) cannot be done here: flagged.
        if (p.k_new != nullptr && part == 0 && len > 0 && start >= nblk && threadIdx.x == 0 &&
            (!MMA || by % p.chunks == 0))
            flag(p.err, PKV_DEV_ERR_BAD_LEN);
        if (!SPLIT)
            for (int i = threadIdx.x; i < heads * D; i += NW * 32)
                p.out[(static_cast<size_t>(b) * p.Hq + h0 + i / D) * D + i % D] = __float2bfloat16(0.f);
        return;
    }

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

    const int n_mine = blk_end - blk_begin > lead ? (blk_end - blk_begin - lead + kStride - 1) / kStride : 0;
    if (!early_table) {
        tw.first = blk_begin + lead;
        tw.count = n_mine;
        tw.init(lane);
    }
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

    // The fused write step: the warp that will read the sequence's last block
    // stores the step's new K and V (position len - 1) into their slot, just
    // before it issues that block's load -- the value is fetched into
    // registers now, the store and the proxy fence (then __syncwarp, so lane
    // 0's TMA read is ordered after them) wait until then.  Several
    // head-chunk CTAs of one KV head store the same bytes.
    const int last_local = nblk - 1 - blk_begin;
    const bool writer = p.k_new != nullptr && blk_end == nblk && len > 0 && warp == last_local % NW;
    const int i_write = last_local / kStride;
    uint4 new_val = make_uint4(0, 0, 0, 0);
    __nv_bfloat16 *new_dst = nullptr;
    if (writer && lane < 2 * (D / 8)) {
        const int pos = len - 1;
        const int32_t phys = __ldg(p.block_tables + static_cast<size_t>(b) * p.W + pos / kBlockTokens);
        if (phys >= 0 && phys < p.num_blocks) {
            const bool is_v = lane >= D / 8;
            const int e = (lane % (D / 8)) * 8;
            new_val = __ldg(reinterpret_cast<const uint4 *>(
                (is_v ? p.v_new : p.k_new) + (static_cast<size_t>(b) * p.Hkv + kvh) * D + e));
            new_dst = (is_v ? p.v_cache : p.k_cache) +
                      ((static_cast<size_t>(phys) * p.Hkv + kvh) * kBlockTokens + pos % kBlockTokens) * D + e;
        }
    }
    auto store_new = [&]() {  // warp-uniform: all lanes of the writer warp
        if (new_dst != nullptr) {
            *reinterpret_cast<uint4 *>(new_dst) = new_val;
            fence_proxy_async_global();
        }
        __syncwarp();
    };

    for (int i = 0; i < S && i < n_mine; ++i) {
        if (writer && i == i_write) store_new();
        issue(i);
    }

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
            const int lb = blk_begin + lead + kStride * i;
            const int nvalid = min(kBlockTokens, len - lb * kBlockTokens);
            const uint8_t *kt = ring + s * G::kStageBytes;
            if constexpr (MMA)
                st.tile(smem_u32(kt), smem_u32(kt + G::kTileBytes), nvalid, lane);
            else
                st.tile(kt, kt + G::kTileBytes, nvalid, lane);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (i + S < n_mine) {
            if (writer && i + S == i_write) store_new();
            issue(i + S);
        }
    }
    if (i < n_mine) {
        // A wait gave up: let the copies still in flight land before the
        // shared memory is reused or released (again bounded).
        for (int j = i; j < n_mine && j < i + S; ++j)
            mbar_wait(bars + 8 * (j % S), static_cast<uint32_t>((j / S) & 1), kWaitLimitNs);
    }

    constexpr int kRed = MMA ? 16 + 8 * D : D + 2;
    // ---- combine the warps of this CTA (all rings are drained) ----
    __syncthreads();
    float *red = reinterpret_cast<float *>(smem);
    // cluster mode: this CTA's combined rows for the other CTAs of the
    // cluster -- m of head n at [n], l at [8 + n], o at [16 + n * D + e]
    float *xch = red + NW * kRed;
    st.finish(red + warp * kRed, lane);
    __syncthreads();
    if constexpr (CLUSTER) {
        if (blk_begin >= blk_end && p.k_new != nullptr && len > 0 && start >= nblk && part == 0 &&
            threadIdx.x == 0 && (!MMA || by % p.chunks == 0))
            flag(p.err, PKV_DEV_ERR_BAD_LEN);  // the fused write's token lies inside the skipped prefix
    }
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
        } else if constexpr (CLUSTER) {
            xch[16 + n * D + e] = O;
            if (e == 0) {
                xch[n] = M;
                xch[8 + n] = L;
            }
        } else {
            p.out[row * D + e] = __float2bfloat16(L > 0.f ? O / L : 0.f);
        }
    }
    if constexpr (CLUSTER) {
        // Log-sum-exp merge of the cluster's parts, in part order (the same
        // arithmetic as the split-K merge kernel): each CTA merges an equal
        // slice of the (head, column) elements, reading every part's m, l and
        // o from the owning CTA's shared memory.
        cluster_sync();
        const int P = p.num_parts;
        const int total = heads * D;
        const int per = (total + P - 1) / P;
        const int lo = static_cast<int>(cluster_ctarank()) * per, hi = min(total, lo + per);
        for (int idx = lo + threadIdx.x; idx < hi; idx += NW * 32) {
            const int n = idx / D, e = idx % D;
            // every part's m, l and o requested at once (one round trip through
            // the cluster), then combined in part order
            float mc[kMaxClusterParts], lc[kMaxClusterParts], oc[kMaxClusterParts];
#pragma unroll
            for (int c = 0; c < kMaxClusterParts; ++c) {
                mc[c] = c < P ? ld_dsmem_f32(xch + n, c) : -INFINITY;
                lc[c] = c < P ? ld_dsmem_f32(xch + 8 + n, c) : 0.f;
                oc[c] = c < P ? ld_dsmem_f32(xch + 16 + n * D + e, c) : 0.f;
            }
            float M = -INFINITY;
#pragma unroll
            for (int c = 0; c < kMaxClusterParts; ++c) M = fmaxf(M, mc[c]);
            float L = 0.f, O = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int c = 0; c < kMaxClusterParts; ++c) {
                    if (c >= P) break;
                    const float wgt = mc[c] == -INFINITY ? 0.f : exp2f(mc[c] - M);
                    L = fmaf(lc[c], wgt, L);
                    O = fmaf(oc[c], wgt, O);
                }
            }
            p.out[(static_cast<size_t>(b) * p.Hq + h0 + n) * D + e] =
                __float2bfloat16(L > 0.f ? O / L : 0.f);
        }
        cluster_sync();  // no CTA leaves while the others still read its shared memory
    }
}

}  // namespace dev
}  // namespace pkv
