// Shared-prefix ("cascade") decode attention.
//
// Several sequences whose block tables start with the same physical blocks
// ("vLLM 與 PagedAttention：高吞吐推理的關鍵", section 二, 無法共享: the tables of
// requests with a common prefix point at one set of blocks) need the same
// prefix K/V.  Plain decode streams those shared blocks once per sequence;
// here they are read once per (group, KV head) and the attention of every
// member's query against them is computed as one dense product -- rows =
// (member, query head of this KV head) pairs, 128 per tile, against a span
// of the prefix's keys -- on the tcgen05 tensor cores with the products in
// TMEM (prefix_unit_tc below); with 128 members that is a 128-row tile per KV
// head, a real dense contraction.  (A warp-level mma.sync version measured
// 1-2.5 % slower per step beside the suffix stream.)  Each prefix CTA takes a
// span of SB prefix blocks, streams its K and V once by TMA in steps of 64
// keys, and leaves one partial (m, l, o) per row.  The private suffixes go
// through the split-K kernel starting past the prefix, and the merge below
// combines prefix and suffix partials of each (sequence, query head) by
// log-sum-exp.  The result equals plain decode over the whole sequence.
#include <algorithm>

#include "decode_unit.cuh"
#include "tcgen05.cuh"

namespace pkv {

namespace {

using namespace dev;

constexpr int kPrefixWarps = 4;

template <int D, int SB>
struct PrefixTcGeometry {
    static constexpr int kSubKeys = 64;                       // keys per step: MMA N of S, K of P.V
    static constexpr int kSubBlocks = kSubKeys / kBlockTokens;
    static constexpr int kSub = (D / 64) * kSubKeys * 128;    // one K or V step tile [d half][key][128 B]
    static constexpr int kStage = 2 * kSub;                   // K then V
    static constexpr int kRing = 2 * kStage;                  // two stages
    static constexpr int kMeta = 64 + 4 * SB;                 // 3 mbarriers, TMEM base, keep bits, rows[SB]
    static constexpr int kSmemBytes = kRing + kMeta + 1024;
    static constexpr int kTmemCols = 256;                     // S (P over its first half) | O | Q
    static constexpr int kColS = 0, kColO = kSubKeys, kColQ = kSubKeys + D;
    static_assert(SB % kSubBlocks == 0 && SB <= 64, "span layout");
    static_assert(kColQ + D / 2 <= kTmemCols, "tensor memory columns");
    static_assert(kRing >= 128 * D * 4, "a row tile's partials staged through the ring");
};

// Prefix span c (blocks [c*SB, (c+1)*SB) of group g's shared prefix) for KV
// head kvh on the tcgen05 tensor cores.  The rows, (member, query head)
// pairs, go in tiles of 128, one row per thread (= TMEM lane); each row
// tile's Q stays in TMEM while the span's keys stream by in steps of 64
// (K and V of a step by TMA into one of two shared-memory stages, the step
// two ahead loaded as soon as a stage is free):
//   S[128 x 64] = Q K^T    tcgen05.mma, A = Q from TMEM, K from shared memory
//   m = running max (moved only when it grows by more than 2^8; O and l
//       rescaled then), P = 2^(S * scale - m) as bf16 into TMEM over S,
//   l += sum P (fp32)
//   O[128 x d] += P V      tcgen05.mma, A = P from TMEM, V from shared memory
// and the row's partial (m, l, O) goes to its workspace slot.  Keys of blocks
// past the prefix or with a bad table entry are loaded as zeros (a row past
// the tensor) and masked to -inf.  Every wait is bounded; on a timeout the
// CTA flags it, waits (bounded) for its copies and MMAs, and frees its TMEM.
template <int D, int SB>
__device__ __forceinline__ void prefix_unit_tc(const CUtensorMap &tmk, const CUtensorMap &tmv,
                                            const PrefixParams &p, int c, int kvh, int g) {
    using Geo = PrefixTcGeometry<D, SB>;
    constexpr int kSubKeys = Geo::kSubKeys, kSubBlocks = Geo::kSubBlocks;
    constexpr int kColS = Geo::kColS, kColO = Geo::kColO, kColQ = Geo::kColQ;
    constexpr uint32_t kIdS = tc::idesc_bf16(128, kSubKeys, 0);
    constexpr uint32_t kIdO = tc::idesc_bf16(128, D, 1);
    constexpr float kRescale = 8.0f;  // log2 units
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;

    const int off = __ldg(p.group_offsets + g);
    const int members = __ldg(p.group_offsets + g + 1) - off;
    if (members <= 0) return;
    const int b0 = __ldg(p.group_seqs + off);
    if (b0 < 0 || b0 >= p.B) {
        if (t == 0) flag(p.err, PKV_DEV_ERR_BAD_LEN);
        return;
    }
    int len0 = __ldg(p.seq_lens + b0);
    len0 = len0 < 0 ? 0 : min(len0, p.W * kBlockTokens);
    const int nb = min(max(__ldg(p.prefix_blocks + b0), 0), len0 / kBlockTokens);  // full blocks
    const int j0 = c * SB, j1 = min(nb, j0 + SB);
    if (j0 >= j1) return;
    const int n_sub = (j1 - j0 + kSubBlocks - 1) / kSubBlocks;  // key steps of the span

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t ring = smem_u32(smem);
    const uint32_t bars = smem_u32(smem + Geo::kRing);
    const auto kv_full = [&](int st) { return bars + 8 * st; };  // a stage's K and V landed
    const uint32_t m_bar = bars + 16;                             // the MMAs issued so far are done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Geo::kRing + 24);
    uint32_t *keep_slot = reinterpret_cast<uint32_t *>(smem + Geo::kRing + 32);  // [2]: blocks 0-31, 32-63
    int *rows = reinterpret_cast<int *>(smem + Geo::kRing + 64);  // [SB] tensor-map row of each block

    if (warp == 0) {  // lane i: blocks j0 + i and j0 + 32 + i of the span
        const int32_t *trow = p.block_tables + static_cast<size_t>(b0) * p.W;
        const int y_none = static_cast<int>(p.num_blocks * p.Hkv * kBlockTokens);  // past the tensor: zeros
#pragma unroll
        for (int hw = 0; hw < 2; ++hw) {
            const int blk = 32 * hw + lane;
            bool ok_blk = false;
            if (blk < SB) {
                int y = y_none;
                if (j0 + blk < j1) {
                    const int32_t phys = __ldg(trow + j0 + blk);
                    if (phys >= 0 && phys < p.num_blocks) {
                        y = (phys * p.Hkv + kvh) * kBlockTokens;
                        ok_blk = true;
                    } else {
                        flag(p.err, PKV_DEV_ERR_BAD_BLOCK);
                    }
                }
                rows[blk] = y;
            }
            const uint32_t bits = __ballot_sync(0xffffffffu, ok_blk);
            if (lane == 0) keep_slot[hw] = bits;
        }
        if (lane == 0) {
            mbar_init(kv_full(0), 1);
            mbar_init(kv_full(1), 1);
            mbar_init(m_bar, 1);
            fence_mbar_init();
            prefetch_tmap(&tmk);
            prefetch_tmap(&tmv);
        }
    }
    if (warp == 1) tc::alloc<Geo::kTmemCols>(smem_u32(tmem_slot));
    tc::fence_before();
    __syncthreads();  // barriers, rows[], keep bits and the TMEM base
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t keep = static_cast<uint64_t>(keep_slot[0]) | (static_cast<uint64_t>(keep_slot[1]) << 32);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);  // this thread's lane
    const uint64_t policy = l2_policy_evict_first();

    // Key step i of the span into stage st ([d half][key][128 B] for K, then V).
    const auto issue_step = [&](int i, int st) {  // thread 0
        const uint32_t kdst = ring + st * Geo::kStage, vdst = kdst + Geo::kSub;
        mbar_arrive_expect_tx(kv_full(st), Geo::kStage);
#pragma unroll
        for (int bb = 0; bb < kSubBlocks; ++bb) {
            const int y = rows[i * kSubBlocks + bb];
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh) {
                tma_load_2d(kdst + hh * (kSubKeys * 128) + bb * (kBlockTokens * 128), &tmk, hh * 64, y,
                            kv_full(st), policy);
                tma_load_2d(vdst + hh * (kSubKeys * 128) + bb * (kBlockTokens * 128), &tmv, hh * 64, y,
                            kv_full(st), policy);
            }
        }
    };

    const int G = p.group;      // query heads per KV head
    const int R = members * G;  // rows of this group and KV head
    bool ok = true;
    bool mma_pending = false;   // an MMA batch committed to m_bar and not yet seen done
    uint32_t phase = 0;         // m_bar phase
    int g_issued = 0, g_landed = 0;  // key-step loads issued / seen landed (stage = n & 1)
    for (int r0 = 0; r0 < R && ok; r0 += 128) {
        if (t == 0)
            for (int i = 0; i < 2 && i < n_sub; ++i) issue_step(i, (g_issued++) & 1);
        const int r = r0 + t;
        int b = -1, h = 0;
        if (r < R) {
            const int bb = __ldg(p.group_seqs + off + r / G);
            if (bb >= 0 && bb < p.B) {
                b = bb;
                h = kvh * G + r % G;
            }
        }
        // Q row -> TMEM columns [kColQ, kColQ + D / 2), zeros for rows without
        // a sequence; all of the row's loads in flight before the stores
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.q + (static_cast<size_t>(b < 0 ? 0 : b) * p.Hq + h) * D);
            uint32_t w[D / 2];
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
                const uint4 v = b >= 0 ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
                w[4 * i] = v.x;
                w[4 * i + 1] = v.y;
                w[4 * i + 2] = v.z;
                w[4 * i + 3] = v.w;
            }
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc) tc::st32(lane_base + kColQ + 32 * cc, w + 32 * cc);
            tc::wait_st();
        }
        tc::fence_before();
        float m_run = -INFINITY, l_run = 0.f;
        for (int i = 0; i < n_sub; ++i) {
            const int st = g_landed & 1;
            if (__syncthreads_or(!mbar_wait(kv_full(st), static_cast<uint32_t>((g_landed >> 1) & 1),
                                            kWaitLimitNs))) {
                ok = false;
                break;
            }
            ++g_landed;
            tc::fence_after();
            const uint32_t kbase = ring + st * Geo::kStage, vbase = kbase + Geo::kSub;
            if (t == 0) {  // S = Q K^T
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    tc::mma_ts(tmem + kColS, tmem + kColQ + 8 * k,
                               tc::smem_desc(kbase + (k >> 2) * (kSubKeys * 128) + (k & 3) * 32, 16, 1024),
                               kIdS, k > 0);
                tc::commit(m_bar);
            }
            mma_pending = true;
            if (__syncthreads_or(!mbar_wait(m_bar, phase, kWaitLimitNs))) {
                ok = false;
                break;
            }
            mma_pending = false;
            phase ^= 1;
            tc::fence_after();

            // softmax of the row over the step's 64 keys (4 blocks)
            const uint32_t kbits = static_cast<uint32_t>(keep >> (i * kSubBlocks));
            uint32_t sv[64];
            tc::ld32(lane_base + kColS, sv);
            tc::ld32(lane_base + kColS + 32, sv + 32);
            tc::wait_ld();
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // one chain per block
#pragma unroll
            for (int k = 0; k < 64; ++k)
                if (kbits >> (k / kBlockTokens) & 1u)
                    mx4[k / kBlockTokens] = fmaxf(mx4[k / kBlockTokens], __uint_as_float(sv[k]) * p.scale_log2);
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            const bool grow = mx > m_run + kRescale || (m_run == -INFINITY && mx != -INFINITY);
            const float m_new = grow ? mx : m_run;
            if (grow && m_run != -INFINITY) {  // O (the previous steps' P.V, done) and l follow the max
                const float alpha = exp2f(m_run - m_new);
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    tc::ld32(lane_base + kColO + 32 * cc, o);
                    tc::wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                    tc::st32(lane_base + kColO + 32 * cc, o);
                }
                l_run *= alpha;
            }
            m_run = m_new;
            const float nbase = m_new == -INFINITY ? 0.f : m_new;
            float l4[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[32];
#pragma unroll
            for (int k = 0; k < 64; k += 2) {
                const bool there = kbits >> (k / kBlockTokens) & 1u;  // k, k + 1: one block
                const float p0 = there ? ex2_approx(fmaf(__uint_as_float(sv[k]), p.scale_log2, -nbase)) : 0.f;
                const float p1 = there ? ex2_approx(fmaf(__uint_as_float(sv[k + 1]), p.scale_log2, -nbase)) : 0.f;
                l4[k / kBlockTokens] += p0 + p1;
                pk[k / 2] = pack_bf16x2(p0, p1);
            }
            l_run += (l4[0] + l4[1]) + (l4[2] + l4[3]);
            tc::st32(lane_base + kColS, pk);  // P over S columns already read
            tc::wait_st();
            tc::fence_before();
            __syncthreads();  // every row's P (and O, when rescaled) in TMEM
            tc::fence_after();
            if (t == 0) {  // O (+)= P V (V MN-major: d contiguous)
#pragma unroll
                for (int k = 0; k < kSubKeys / 16; ++k)
                    tc::mma_ts(tmem + kColO, tmem + kColS + 8 * k,
                               tc::smem_desc(vbase + k * (16 * 128), kSubKeys * 128, 1024), kIdO,
                               i > 0 || k > 0);
                tc::commit(m_bar);
            }
            mma_pending = true;
            if (__syncthreads_or(!mbar_wait(m_bar, phase, kWaitLimitNs))) {
                ok = false;
                break;
            }
            mma_pending = false;
            phase ^= 1;
            tc::fence_after();
            // the stage is free: the step two ahead
            if (t == 0 && i + 2 < n_sub) issue_step(i + 2, (g_issued++) & 1);
        }
        if (!ok) break;

        // the row's partial for span c
        const size_t slot = (static_cast<size_t>(b < 0 ? 0 : b) * p.Hq + h) * p.ws_parts + c;
        if (b >= 0) {
            p.ws_ml[2 * slot] = m_run;
            p.ws_ml[2 * slot + 1] = l_run;
        }
        if (R <= 128) {
            // The only row tile: the ring is no longer read, so the rows go
            // through it ([row][D floats], 16-byte chunk j of row t at
            // j ^ (t % chunks per row)) and each warp then writes its lanes'
            // rows whole, one 16-byte chunk per lane.
            constexpr int kChunks = D / 4;  // 16-byte chunks of a row
            float4 *stage = reinterpret_cast<float4 *>(smem);
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tc::ld32(lane_base + kColO + 32 * cc, o);
                tc::wait_ld();
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    stage[t * kChunks + ((8 * cc + i) ^ (t & (kChunks - 1)))] =
                        make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                    __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
            }
            __syncwarp();  // a warp writes out its own lanes' rows
#pragma unroll 1
            for (int i = 0; i < 32; ++i) {
                const int rr = 32 * warp + i;
                const unsigned long long rslot = __shfl_sync(0xffffffffu, static_cast<unsigned long long>(slot), i);
                if (!__shfl_sync(0xffffffffu, b >= 0, i)) continue;
                float4 *rdst = reinterpret_cast<float4 *>(p.ws_o + rslot * D);
                for (int j = lane; j < kChunks; j += 32)
                    rdst[j] = stage[rr * kChunks + (j ^ (rr & (kChunks - 1)))];
            }
        } else {
            float4 *dst = reinterpret_cast<float4 *>(p.ws_o + slot * D);
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tc::ld32(lane_base + kColO + 32 * cc, o);
                tc::wait_ld();
                if (b >= 0) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[8 * cc + i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                                      __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
                }
            }
            tc::fence_before();
            __syncthreads();  // O read by every thread before the next row tile's P.V
            tc::fence_after();
        }
    }
    if (!ok && t == 0) {
        flag(p.err, PKV_DEV_ERR_TIMEOUT);
        if (mma_pending) mbar_wait(m_bar, phase, kWaitLimitNs);  // the batch still running
    }
    if (t == 0)  // copies still landing (none unless a wait gave up)
        for (int n = g_landed; n < g_issued; ++n)
            mbar_wait(kv_full(n & 1), static_cast<uint32_t>((n >> 1) & 1), kWaitLimitNs);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 1) tc::dealloc<Geo::kTmemCols>(tmem);
}

// Merge of one (sequence, query head): prefix spans [0, ceil(pb / CB)) and
// the suffix split-K partitions that hold tokens past the prefix (counted
// from the prefix end), in slot order, by log-sum-exp.  One warp per row,
// kMergeRows rows per CTA, so that the whole merge grid is resident at once
// (a CTA of D threads per row made two waves of short CTAs at batch 128,
// 32 heads); lane l holds columns [l V, l V + V).  A lane reads the (m, l)
// of one slot, the warp reduces them, then every slot's o is loaded 8 slots
// at a time and accumulated in slot order.
constexpr int kMergeRows = 4;

template <int D, int CB>
__global__ void __launch_bounds__(kMergeRows * 32) cascade_merge_kernel(const PrefixParams p) {
    constexpr int V = D / 32;  // columns per lane
    pdl_launch_dependents();  // the next call's first grid may be scheduled
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * kMergeRows + warp;  // row = b * Hq + h
    const bool live = r < p.B * p.Hq;
    const int b = live ? r / p.Hq : 0;
    // the slot count comes from the step's inputs, read before the wait
    int len = __ldg(p.seq_lens + b);
    len = len < 0 ? 0 : min(len, p.W * kBlockTokens);
    const int nblk = (len + kBlockTokens - 1) / kBlockTokens;
    const int pb = min(max(__ldg(p.prefix_blocks + b), 0), len / kBlockTokens);
    const int nchunks = (pb + CB - 1) / CB;  // prefix spans
    // suffix partitions with tokens, at most those the launch computed (a
    // longer suffix was flagged by the cascade kernel)
    const int ntot = nchunks + min((nblk - pb + p.part_blocks - 1) / p.part_blocks,
                                   p.ws_parts - p.prefix_parts);
    const auto slot = [&](int q) { return q < nchunks ? q : p.prefix_parts + (q - nchunks); };
    const size_t row = static_cast<size_t>(live ? r : 0);
    const float *ml = p.ws_ml + 2 * row * p.ws_parts;
    const float *o = p.ws_o + row * p.ws_parts * D + lane * V;
    pdl_wait_primary();  // the cascade grid's partials
    if (!live) return;
    float M = -INFINITY;
    for (int q = lane; q < ntot; q += 32) M = fmaxf(M, ml[2 * slot(q)]);
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    float L = 0.f, O[V];
#pragma unroll
    for (int v = 0; v < V; ++v) O[v] = 0.f;
    if (M != -INFINITY) {
        for (int q0 = 0; q0 < ntot; q0 += 32) {
            // weight of slot q0 + lane, then the slots' o in order
            float w = 0.f, lq = 0.f;
            if (q0 + lane < ntot) {
                const float2 v = *reinterpret_cast<const float2 *>(ml + 2 * slot(q0 + lane));
                w = v.x == -INFINITY ? 0.f : exp2f(v.x - M);
                lq = v.y * w;
            }
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) lq += __shfl_xor_sync(0xffffffffu, lq, m);
            L += lq;
            const int n = min(32, ntot - q0);
            for (int k0 = 0; k0 < n; k0 += 8) {
                float x[8][V];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (k0 + k < n) {
                        const float *src = o + static_cast<size_t>(slot(q0 + k0 + k)) * D;
                        if constexpr (V == 4) {
                            const float4 t = *reinterpret_cast<const float4 *>(src);
                            x[k][0] = t.x;
                            x[k][1] = t.y;
                            x[k][2] = t.z;
                            x[k][3] = t.w;
                        } else {
                            const float2 t = *reinterpret_cast<const float2 *>(src);
                            x[k][0] = t.x;
                            x[k][1] = t.y;
                        }
                    }
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float wk = __shfl_sync(0xffffffffu, w, (k0 + k) & 31);
                    if (k0 + k < n) {
#pragma unroll
                        for (int v = 0; v < V; ++v) O[v] = fmaf(x[k][v], wk, O[v]);
                    }
                }
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16 *dst = p.out + row * D + lane * V;
#pragma unroll
    for (int v = 0; v < V; v += 2)
        *reinterpret_cast<__nv_bfloat162 *>(dst + v) = __floats2bfloat162_rn(O[v] * inv, O[v + 1] * inv);
}

// One launch for the prefix spans and the suffix split-K units.  Prefix
// span k (span fastest, then KV head, then group) is CTA k * stride, spread
// evenly through the first eighth of the grid, so that the latency-bound
// prefix work runs beside the bandwidth-bound suffix stream and its long
// CTAs (a span of up to 1024 keys) are done well before the stream is
// (spread over the whole grid, the last spans started late and ended after
// it: 119.5 against 109.8 us per step with 32-block spans); the other CTAs
// take suffix units in order (partition fastest, then head segment, then
// sequence).
template <int D, bool MMA>
__global__ void __launch_bounds__(kPrefixWarps * 32, 3)  // three CTAs per SM, as the suffix units need
    cascade_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                   const PrefixParams pp, const DecodeParams dp, int n_pre) {
    pdl_launch_dependents();
    int id = blockIdx.x;
    const int stride = n_pre > 0 ? max(1, static_cast<int>(gridDim.x) / 8 / n_pre) : 1;
    if (n_pre > 0 && id % stride == 0 && id / stride < n_pre) {
        pdl_wait_primary();  // the previous call's grid
        id /= stride;
        const int c = id % pp.prefix_parts;
        id /= pp.prefix_parts;
        prefix_unit_tc<D, kPrefixSpanBlocks>(tmk, tmv, pp, c, id % pp.Hkv, id / pp.Hkv);
        return;
    }
    // Suffix units use no TMEM: they give up the right to allocate at once.
    // A CTA that keeps it (until it exits) holds up the TMEM allocation of a
    // prefix CTA that starts after it on the same SM (measured: the step took
    // twice as long).
    if (n_pre > 0 && threadIdx.x < 32) tc::relinquish();
    if (n_pre > 0) id -= min(id / stride + 1, n_pre);  // prefix CTAs at or before this one
    const int ny = MMA ? dp.Hkv * dp.chunks : dp.Hq;
    const int part = id % dp.num_parts;
    id /= dp.num_parts;
    const int b = id / ny;
    if (part == dp.num_parts - 1 && id % ny == 0 && threadIdx.x == 0 && b < dp.B) {
        // the caller's bound on suffix blocks must cover every suffix
        int len = __ldg(dp.seq_lens + b);
        len = len < 0 ? 0 : min(len, dp.W * kBlockTokens);
        const int start = min(max(__ldg(dp.start_blocks + b), 0), len / kBlockTokens);
        if (start + dp.num_parts * dp.part_blocks < (len + kBlockTokens - 1) / kBlockTokens)
            flag(dp.err, PKV_DEV_ERR_BAD_LEN);
    }
    // the unit reads the length, start block and table row, then waits for the
    // previous call's grid before anything that grid may write
    decode_unit<D, kPrefixWarps, 2, MMA, kModeSplit>(tmk, tmv, dp, part, id % ny, b, true);
}

template <int D, bool MMA>
cudaError_t launch_cascade_d(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefixParams &pp,
                             const DecodeParams &dp, int num_groups, cudaStream_t stream) {
    constexpr int kPre = PrefixTcGeometry<D, kPrefixSpanBlocks>::kSmemBytes;
    constexpr int kSmem = std::max(kPre, Geometry<D, kPrefixWarps, 2>::kSmemBytes);
    auto kern = cascade_kernel<D, MMA>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    const long long n_pre = static_cast<long long>(pp.prefix_parts) * pp.Hkv * num_groups;
    const long long ny = MMA ? dp.Hkv * dp.chunks : dp.Hq;
    const long long n_suf = static_cast<long long>(dp.num_parts) * ny * dp.B;
    if (n_pre + n_suf >= (1ll << 31)) return cudaErrorInvalidValue;
    e = launch_dependent_smem(kern, dim3(static_cast<unsigned>(n_pre + n_suf)), dim3(kPrefixWarps * 32),
                              kSmem, stream, tmk, tmv, pp, dp, static_cast<int>(n_pre));
    if (e != cudaSuccess) return e;
    const long long rows = static_cast<long long>(pp.B) * pp.Hq;
    return launch_dependent(cascade_merge_kernel<D, kPrefixSpanBlocks>,
                            dim3(static_cast<unsigned>((rows + kMergeRows - 1) / kMergeRows)),
                            dim3(kMergeRows * 32), stream, pp);
}

template <int D>
cudaError_t launch_cascade_h(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefixParams &pp,
                             const DecodeParams &dp, int num_groups, cudaStream_t stream) {
    return dp.group > 1 ? launch_cascade_d<D, true>(tmk, tmv, pp, dp, num_groups, stream)
                        : launch_cascade_d<D, false>(tmk, tmv, pp, dp, num_groups, stream);
}

}  // namespace

cudaError_t launch_cascade(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefixParams &pp,
                           const DecodeParams &dp, int head_dim, int num_groups, cudaStream_t stream) {
    if (head_dim == 128) return launch_cascade_h<128>(tmk, tmv, pp, dp, num_groups, stream);
    if (head_dim == 64) return launch_cascade_h<64>(tmk, tmv, pp, dp, num_groups, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pkv
