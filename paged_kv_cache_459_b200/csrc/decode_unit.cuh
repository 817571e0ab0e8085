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

// Cluster mode: the shared memory of part 0 past its ring and barriers takes
// an mbarrier (16 bytes with padding) and, with one query head per CTA, the
// combined rows of parts 1 .. P - 1, each [m of <= H heads][l of <= H
// heads][o: H x D] floats, so that they can arrive while part 0 still reads
// its own blocks.  With a group of heads (8 x the rows) they go into part 0's
// ring instead, behind its own rows, once part 0 has passed a cluster barrier
// after its blocks (three CTAs per SM either way).
template <int D, bool MMA>
constexpr int cluster_slot_floats() {
    return (MMA ? 8 : 1) * (D + 2);
}
template <bool MMA>
constexpr bool cluster_land_in_ring() {
    return MMA;
}
template <int D, bool MMA>
constexpr int cluster_land_bytes() {
    return 16 + (cluster_land_in_ring<MMA>() ? 0 : (kMaxClusterParts - 1) * cluster_slot_floats<D, MMA>() * 4);
}

// One work unit (partition `part` of sequence b, KV head / head chunk `by`)
// of the per-unit decode kernel, run by a CTA of NW warps.  The warps take
// the unit's blocks round-robin and are combined in shared memory at the end.
template <int D, int NW, int S, bool MMA, int MODE>
__device__ __forceinline__ void decode_unit(const CUtensorMap &tmk, const CUtensorMap &tmv,
                                            const DecodeParams &p, int part, int by, int b,
                                            bool wait_pending = false) {
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
        if (wait_pending) pdl_wait_primary();
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
    // Cluster mode: parts 1 .. P - 1 store their combined rows into part 0's
    // shared memory and arrive on its mbarrier `land`; part 0 merges.  A
    // cluster barrier whose wait comes before the first store makes the
    // mbarrier's initialisation visible to the other parts; it starts here
    // when the rows land outside part 0's ring, else after each part's blocks.
    const int P = CLUSTER ? p.num_parts : 1;
    const uint32_t land = smem_u32(smem + G::kRingBytes + NW * S * 8);
    uint32_t rank = 0;
    if constexpr (CLUSTER) {
        rank = cluster_ctarank();
        if (P > 1 && rank == 0 && threadIdx.x == 0) {
            mbar_init(land, P - 1);
            fence_mbar_init();
        }
    }
    __syncthreads();
    if constexpr (CLUSTER) {
        if (P > 1 && !cluster_land_in_ring<MMA>()) cluster_arrive_release();
    }

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

    // The lengths and the table row (host-written metadata) were read above;
    // everything from here on -- q, the new token, K/V, the outputs -- may be
    // the preceding grid's, so the wait for it comes first.
    if (wait_pending) pdl_wait_primary();
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
    constexpr int kHeadsMax = MMA ? 8 : 1;
    constexpr int kSlot = cluster_slot_floats<D, MMA>();
    // ---- combine the warps of this CTA (all rings are drained) ----
    __syncthreads();
    float *red = reinterpret_cast<float *>(smem);
    // cluster mode, part 0: its own combined rows -- m of head n at [n], l at
    // [8 + n], o at [16 + n * D + e]
    float *xch = red + NW * kRed;
    st.finish(red + warp * kRed, lane);
    __syncthreads();
    uint32_t my_slot = 0;  // cluster mode, parts 1 .. P - 1: this part's rows in part 0
    // where the other parts' rows land in part 0: behind xch in the ring, or
    // behind the mbarrier
    const uint32_t land_rows = cluster_land_in_ring<MMA>()
                                   ? (smem_u32(xch + 16 + 8 * D) + 15u) & ~15u
                                   : land + 16;
    static_assert(!CLUSTER || !cluster_land_in_ring<MMA>() ||
                      (NW * kRed + 16 + 8 * D + 4) * 4 + (kMaxClusterParts - 1) * kSlot * 4 <= G::kRingBytes,
                  "the other parts' rows must fit in part 0's ring");
    if constexpr (CLUSTER) {
        if (blk_begin >= blk_end && p.k_new != nullptr && len > 0 && start >= nblk && part == 0 &&
            threadIdx.x == 0 && (!MMA || by % p.chunks == 0))
            flag(p.err, PKV_DEV_ERR_BAD_LEN);  // the fused write's token lies inside the skipped prefix
        if (P > 1) {
            if (cluster_land_in_ring<MMA>()) cluster_arrive_release();  // this part's blocks are read
            cluster_wait_acquire();  // part 0's mbarrier is initialised (and its ring free)
            if (rank != 0) my_slot = dsmem_addr(land_rows + (rank - 1) * kSlot * 4, 0);
        }
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
            if (rank == 0) {
                xch[16 + n * D + e] = O;
                if (e == 0) {
                    xch[n] = M;
                    xch[8 + n] = L;
                }
            } else {
                st_dsmem_f32(my_slot + 4 * (2 * kHeadsMax + n * D + e), O);
                if (e == 0) {
                    st_dsmem_f32(my_slot + 4 * n, M);
                    st_dsmem_f32(my_slot + 4 * (kHeadsMax + n), L);
                }
            }
        } else {
            p.out[row * D + e] = __float2bfloat16(L > 0.f ? O / L : 0.f);
        }
    }
    if constexpr (CLUSTER) {
        if (rank != 0) {
            // every thread's stores are issued; one release at cluster scope
            // covers them, and the part may leave (nothing reads its memory)
            fence_acq_rel_cluster();
            __syncthreads();
            if (threadIdx.x == 0) {
                fence_acq_rel_cluster();
                mbar_arrive_remote(dsmem_addr(land, 0));
            }
            return;
        }
        // Part 0: log-sum-exp merge of the cluster's parts, in part order
        // (the same arithmetic as the split-K merge kernel), its own rows from
        // xch and the others' from its landing area.  The wait outlasts every
        // part's own bounded waits, so no part stores here after part 0 left.
        if (P > 1 && !mbar_wait_cluster(land, 0, kWaitLimitNs * static_cast<uint64_t>(pblk + 4)) &&
            threadIdx.x == 0)
            flag(p.err, PKV_DEV_ERR_TIMEOUT);
        __syncthreads();  // xch complete
        const float *lz = reinterpret_cast<const float *>(smem + (land_rows - smem_u32(smem)));
        for (int idx = threadIdx.x; idx < heads * D; idx += NW * 32) {
            const int n = idx / D, e = idx % D;
            float mc[kMaxClusterParts], lc[kMaxClusterParts], oc[kMaxClusterParts];
            mc[0] = xch[n];
            lc[0] = xch[8 + n];
            oc[0] = xch[16 + n * D + e];
#pragma unroll
            for (int c = 1; c < kMaxClusterParts; ++c) {
                const float *sl = lz + (c - 1) * kSlot;
                mc[c] = c < P ? sl[n] : -INFINITY;
                lc[c] = c < P ? sl[kHeadsMax + n] : 0.f;
                oc[c] = c < P ? sl[2 * kHeadsMax + n * D + e] : 0.f;
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
    }
}

}  // namespace dev
}  // namespace pkv
