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
#include <cfloat>
#include <type_traits>

#include "../../include/pkv.h"
#include "internal.h"
#include "ptx.cuh"

namespace pkv {

namespace {

constexpr uint64_t kWaitLimitNs = 250ull * 1000ull * 1000ull;  // 0.25 s per wait
constexpr int kBoxBytes = 16 * 128;                            // 16 rows x 128 B

// Byte offset of 16-byte chunk `c` of row `r` inside one K or V tile stored
// as head_dim/64 TMA boxes of [16 rows][128 B] with the 128-byte swizzle
// (chunk index XOR row % 8 within each 1024-byte group of 8 rows).
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
    return static_cast<uint32_t>((c >> 3) * kBoxBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void flag(unsigned int *err, unsigned int bit) {
    if (err != nullptr) atomicOr(err, bit);
}

template <int D, int NW, int S>
struct Geometry {
    static constexpr int kHalves = D / 64;
    static constexpr int kTileBytes = kHalves * kBoxBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kRingBytes = NW * S * kStageBytes;
    static constexpr int kSmemBytes = kRingBytes + NW * S * 8 + 1024;  // + barriers + alignment
};

// Block-table entries of one warp's blocks, 32 per register load.
struct TableWindow {
    const int32_t *row;  // this sequence's table row
    int first, stride, count;
    int cur_chunk;
    int32_t cur, nxt;

    __device__ __forceinline__ int32_t load(int i) const {
        return i < count ? __ldg(row + first + stride * i) : -1;
    }
    __device__ __forceinline__ void init(int lane) {
        cur_chunk = 0;
        cur = load(lane);
        nxt = load(32 + lane);
    }
    // Warp-uniform i; i >> 5 is cur_chunk or cur_chunk + 1.
    __device__ __forceinline__ int32_t get(int i) const {
        const int32_t v = (i >> 5) == cur_chunk ? cur : nxt;
        return __shfl_sync(0xffffffffu, v, i & 31);
    }
    __device__ __forceinline__ void advance_to(int i, int lane) {
        if ((i >> 5) != cur_chunk) {
            cur = nxt;
            ++cur_chunk;
            nxt = load(32 * (cur_chunk + 1) + lane);
        }
    }
};

// ----------------------------------------------------------------------------
// Per-warp state and tile math: CUDA-core path (one query row per KV head).
template <int D>
struct ScalarHead {
    static constexpr int CH = D / 8;    // 16-byte chunks per row = lanes per row
    static constexpr int RG = 32 / CH;  // rows covered by one pass of the warp
    static constexpr int RPL = 16 / RG; // rows per lane per tile

    float qf[8];
    float o[8];
    float m_run, l_run;
    int c, g;

    __device__ __forceinline__ void init(const __nv_bfloat16 *qrow, float scale_log2, int lane) {
        c = lane % CH;
        g = lane / CH;
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(qrow) + c);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            qf[2 * i] = bf16lo(w[i]) * scale_log2;
            qf[2 * i + 1] = bf16hi(w[i]) * scale_log2;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = 0.f;
        m_run = -INFINITY;
        l_run = 0.f;
    }

    __device__ __forceinline__ void tile(const uint8_t *kt, const uint8_t *vt, int nvalid, int lane) {
        float acc[RPL];
#pragma unroll
        for (int j = 0; j < RPL; ++j) {
            const int r = g + RG * j;
            const uint4 kv = *reinterpret_cast<const uint4 *>(kt + tile_off(r, c));
            float a = qf[0] * bf16lo(kv.x);
            a = fmaf(qf[1], bf16hi(kv.x), a);
            a = fmaf(qf[2], bf16lo(kv.y), a);
            a = fmaf(qf[3], bf16hi(kv.y), a);
            a = fmaf(qf[4], bf16lo(kv.z), a);
            a = fmaf(qf[5], bf16hi(kv.z), a);
            a = fmaf(qf[6], bf16lo(kv.w), a);
            a = fmaf(qf[7], bf16hi(kv.w), a);
            acc[j] = a;
        }
        // Reduce-scatter over the CH lanes of a row group: after it, lane
        // holds the score of local row (lane % CH) >> 1 (twice per pair).
#pragma unroll
        for (int k = RPL, m = CH / 2; k > 1; k >>= 1, m >>= 1) {
            const bool up = (lane & m) != 0;
#pragma unroll
            for (int t = 0; t < k / 2; ++t) {
                const float keep = up ? acc[t + k / 2] : acc[t];
                const float send = up ? acc[t] : acc[t + k / 2];
                acc[t] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        }
        float s = acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 1);
        const int my_row = g + RG * ((lane % CH) >> 1);
        if (my_row >= nvalid) s = -INFINITY;
        float mx = s;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
        const float m_new = fmaxf(m_run, mx);  // finite: the tile has a valid row
        const float alpha = exp2f(m_run - m_new);
        const float p = exp2f(s - m_new);
        l_run = l_run * alpha + ((lane & 1) ? 0.f : p);
        m_run = m_new;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] *= alpha;
#pragma unroll
        for (int j = 0; j < RPL; ++j) {
            const int r = g + RG * j;
            const float pj = __shfl_sync(0xffffffffu, p, g * CH + 2 * j);
            if (r < nvalid) {  // rows past the end may hold anything, NaN included
                const uint4 vv = *reinterpret_cast<const uint4 *>(vt + tile_off(r, c));
                o[0] = fmaf(pj, bf16lo(vv.x), o[0]);
                o[1] = fmaf(pj, bf16hi(vv.x), o[1]);
                o[2] = fmaf(pj, bf16lo(vv.y), o[2]);
                o[3] = fmaf(pj, bf16hi(vv.y), o[3]);
                o[4] = fmaf(pj, bf16lo(vv.z), o[4]);
                o[5] = fmaf(pj, bf16hi(vv.z), o[5]);
                o[6] = fmaf(pj, bf16lo(vv.w), o[6]);
                o[7] = fmaf(pj, bf16hi(vv.w), o[7]);
            }
        }
    }

    // Writes this warp's (m, l, o[D]) into red (D + 2 floats).
    __device__ __forceinline__ void finish(float *red, int lane) {
#pragma unroll
        for (int m = CH; m < 32; m <<= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] += __shfl_xor_sync(0xffffffffu, o[e], m);
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, m);
        if (lane < CH) {
#pragma unroll
            for (int e = 0; e < 8; ++e) red[c * 8 + e] = o[e];
        }
        if (lane == 0) {
            red[D] = m_run;
            red[D + 1] = l_run;
        }
    }
};

// ----------------------------------------------------------------------------
// Per-warp state and tile math: tensor-core path (a group of query heads).
template <int D>
struct GroupHeads {
    static constexpr int KS = D / 16;  // k-steps of S = K.Q^T, m-tiles of O^T

    uint32_t qb[KS][2];  // Q^T as mma B fragments (bf16, unscaled)
    float o[KS][4];      // O^T accumulators: rows d, columns = heads
    float m_run[2], l_run[2];
    float scale_log2;

    __device__ __forceinline__ void init(const __nv_bfloat16 *q0, int heads, float sl2, int lane) {
        const int tig = lane & 3, gid = lane >> 2;
        const bool ok = gid < heads;
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(q0 + static_cast<size_t>(gid) * D);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            qb[ks][0] = ok ? __ldg(qrow + (16 * ks + 2 * tig) / 2) : 0u;
            qb[ks][1] = ok ? __ldg(qrow + (16 * ks + 8 + 2 * tig) / 2) : 0u;
        }
#pragma unroll
        for (int mt = 0; mt < KS; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) o[mt][i] = 0.f;
        m_run[0] = m_run[1] = -INFINITY;
        l_run[0] = l_run[1] = 0.f;
        scale_log2 = sl2;
    }

    __device__ __forceinline__ void tile(uint32_t kt, uint32_t vt, int nvalid, int lane) {
        const int tig = lane & 3, gid = lane >> 2;
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
            const int cb = lane >> 4;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(kt + tile_off(r, 2 * ks + cb), a0, a1, a2, a3);
                mma_bf16_16816(sc, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
            }
        }
        // sc: [token gid][head 2tig], [gid][2tig+1], [gid+8][2tig], [gid+8][2tig+1]
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[i] *= scale_log2;
        if (gid >= nvalid) sc[0] = sc[1] = -INFINITY;
        if (gid + 8 >= nvalid) sc[2] = sc[3] = -INFINITY;
        float mx0 = fmaxf(sc[0], sc[2]), mx1 = fmaxf(sc[1], sc[3]);
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, m));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, m));
        }
        const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
        const float al0 = exp2f(m_run[0] - mn0), al1 = exp2f(m_run[1] - mn1);
        const float p0 = exp2f(sc[0] - mn0), p1 = exp2f(sc[1] - mn1);
        const float p2 = exp2f(sc[2] - mn0), p3 = exp2f(sc[3] - mn1);
        l_run[0] = l_run[0] * al0 + p0 + p2;
        l_run[1] = l_run[1] * al1 + p1 + p3;
        m_run[0] = mn0;
        m_run[1] = mn1;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
            o[mt][0] *= al0;
            o[mt][1] *= al1;
            o[mt][2] *= al0;
            o[mt][3] *= al1;
        }
        // P^T (tokens x heads) from accumulator layout to B-operand layout.
        const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
        const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));
        // Tokens past the end: V rows there may hold NaN; 0 * NaN would leak.
        uint32_t keep01 = 0xFFFFFFFFu, keep23 = 0xFFFFFFFFu;
        if (nvalid < 16) {
            const int t = 2 * tig;
            keep01 = (t < nvalid ? 0x0000FFFFu : 0u) | (t + 1 < nvalid ? 0xFFFF0000u : 0u);
            keep23 = (t + 8 < nvalid ? 0x0000FFFFu : 0u) | (t + 9 < nvalid ? 0xFFFF0000u : 0u);
        }
        const int tok = (lane & 7) + (lane >> 4) * 8;
        const int cb = (lane >> 3) & 1;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
            uint32_t v0, v1, v2, v3;
            ldmatrix_x4_trans(vt + tile_off(tok, 2 * mt + cb), v0, v1, v2, v3);
            mma_bf16_16816(o[mt], v0 & keep01, v1 & keep01, v2 & keep23, v3 & keep23, pb0, pb1);
        }
    }

    // Writes this warp's m[8], l[8], o[8][D] into red (16 + 8 * D floats).
    __device__ __forceinline__ void finish(float *red, int lane) {
        const int tig = lane & 3, gid = lane >> 2;
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
            l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], m);
            l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], m);
        }
        float *ro = red + 16;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
            ro[(2 * tig) * D + 16 * mt + gid] = o[mt][0];
            ro[(2 * tig + 1) * D + 16 * mt + gid] = o[mt][1];
            ro[(2 * tig) * D + 16 * mt + gid + 8] = o[mt][2];
            ro[(2 * tig + 1) * D + 16 * mt + gid + 8] = o[mt][3];
        }
        if (gid == 0) {
            red[2 * tig] = m_run[0];
            red[2 * tig + 1] = m_run[1];
            red[8 + 2 * tig] = l_run[0];
            red[8 + 2 * tig + 1] = l_run[1];
        }
    }
};

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
    const int blk_begin = part * p.part_blocks;
    const int blk_end = min(nblk, blk_begin + p.part_blocks);
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
            const size_t pr = row * p.num_parts + part;
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
    const float *ml = p.ws_ml + 2 * row * p.num_parts;
    const float *o = p.ws_o + row * p.num_parts * D;
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
    if (e != cudaSuccess || !SPLIT) return e;
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
