// Balanced ("stream-K") paged decode attention.
//
// Same result as the other decode variants ("vLLM 與 PagedAttention：高吞吐推理的
// 關鍵", section 三 step 三: attention over all earlier K/V looked up through
// the block table), scheduled differently.  All (sequence, KV head [, chunk of
// <= 8 query heads], logical block) tiles are laid out in one flattened order
// -- sequence, then head segment, then block -- and every warp of a persistent
// grid takes an equal contiguous range of it:
//   worker w of G owns tiles [floor(w T / G), floor((w+1) T / G)).
// A worker streams its range through its own TMA ring without ever draining
// it between (sequence, head) segments, so the ring stays full from the
// first tile to the last and no CTA waits for another.  A segment that lies
// inside one worker's range is finished there (normalised, bf16, written to
// `out`).  A segment cut by worker boundaries leaves one partial (m, l, o)
// per piece in the workspace, at slot (worker + segment) -- unique, because
// worker and segment ranges are both monotone in the flattened order -- and
// the worker holding the segment's first tile records which workers hold the
// rest.  A second kernel merges those pieces by log-sum-exp, in worker order.
//
// The producer side of each warp walks the flattened order S tiles ahead of
// the consumer side and hands each stage's metadata (physical block, valid
// tokens, piece boundaries) to the consumer through shared memory, published
// by the same mbarrier arrive that arms the TMA transaction count.
#include "decode_common.cuh"

namespace pkv {

namespace {

using namespace dev;

constexpr int kFlagFirst = 1 << 8;   // first tile of this worker's piece of a segment
constexpr int kFlagLast = 1 << 9;    // last tile of the piece
constexpr int kFlagWhole = 1 << 10;  // the piece is the whole segment
constexpr int kFlagDir = 1 << 11;    // this worker holds the segment's first tile

__device__ __forceinline__ int clamp_len(int len, int W) {
    return len < 0 ? 0 : (len > W * kBlockTokens ? W * kBlockTokens : len);
}

__device__ __forceinline__ long long warp_incl_scan_ll(long long v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const long long t = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += t;
    }
    return v;
}

// Table entries of one sequence, 32 per register load, read ahead one chunk.
struct RowWindow {
    const int32_t *row;
    int count, chunk;
    int32_t cur, nxt;
    __device__ __forceinline__ int32_t load(int j) const { return j < count ? __ldg(row + j) : -1; }
    __device__ __forceinline__ void reset(const int32_t *r, int n, int j, int lane) {
        row = r;
        count = n;
        chunk = j >> 5;
        cur = load(32 * chunk + lane);
        nxt = load(32 * chunk + 32 + lane);
    }
    __device__ __forceinline__ void advance(int j, int lane) {
        if ((j >> 5) != chunk) {
            cur = nxt;
            ++chunk;
            nxt = load(32 * chunk + 32 + lane);
        }
    }
    __device__ __forceinline__ int32_t get(int j) const { return __shfl_sync(0xffffffffu, cur, j & 31); }
};

// Position of the producer in the flattened tile order, with the constants
// of the segment it is in (computed once per segment).
struct Cursor {
    int b, y, j, nblk, len;
    long long seq_f;  // flattened index of tile (b, 0, 0)
    int seg_flags;    // kFlagWhole / kFlagDir for this worker's piece of the segment
    int w_hi;         // worker holding the segment's last tile
};

template <int D, int NW, int S, bool MMA>
__global__ void __launch_bounds__(NW * 32)
    paged_decode_stream_kernel(const __grid_constant__ CUtensorMap tmk,
                               const __grid_constant__ CUtensorMap tmv, const StreamParams p) {
    using Geo = Geometry<D, NW, S>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long G = static_cast<long long>(gridDim.x) * NW;
    const long long w = static_cast<long long>(blockIdx.x) * NW + warp;
    const int Y = p.Y;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = smem + warp * S * Geo::kStageBytes;
    const uint32_t bars = smem_u32(smem + Geo::kRingBytes) + warp * S * 8;
    int4 *meta = reinterpret_cast<int4 *>(smem + Geo::kRingBytes + NW * S * 8) + warp * S;
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bars + 8 * s, 1);
        fence_mbar_init();
    }
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    __syncthreads();

    // ---- total tiles T (one CTA-wide scan of the lengths) and this worker's range ----
    // Thread t sums sequences [t * per, (t + 1) * per); the exclusive prefix of
    // those sums over the CTA is kept in shared memory for the search below.
    long long *s_pref = reinterpret_cast<long long *>(meta + NW * S - warp * S);  // [NW * 32 + 1]
    const int per = (p.B + NW * 32 - 1) / (NW * 32);
    {
        long long mine = 0;
        const int t0 = threadIdx.x * per;
#pragma unroll 4
        for (int i = 0; i < per; ++i) {
            const int b = t0 + i;
            if (b < p.B) {
                const int raw = __ldg(p.seq_lens + b);
                if ((raw < 0 || raw > p.W * kBlockTokens) && blockIdx.x == 0) flag(p.err, PKV_DEV_ERR_BAD_LEN);
                mine += (clamp_len(raw, p.W) + kBlockTokens - 1) / kBlockTokens;
            }
        }
        mine *= Y;
        const long long incl = warp_incl_scan_ll(mine, lane);
        if (lane == 31) s_pref[warp] = incl;  // warp totals, overwritten below
        __syncthreads();
        long long before = 0;
        for (int v = 0; v < warp; ++v) before += s_pref[v];
        long long total = 0;
        for (int v = 0; v < NW; ++v) total += s_pref[v];
        __syncthreads();
        s_pref[threadIdx.x] = before + incl - mine;
        if (threadIdx.x == 0) s_pref[NW * 32] = total;
        __syncthreads();
    }
    const long long T = s_pref[NW * 32];
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.ws_total = T;
    const long long f0 = w * T / G, f1 = (w + 1) * T / G;
    if (f0 >= f1) return;
    const int ntiles = static_cast<int>(f1 - f0);

    // ---- locate tile f0: the thread chunk holding it, then the sequence ----
    Cursor cu;
    {
        int tstar = 0;
        for (int v = lane; v < NW * 32; v += 32)
            if (s_pref[v] <= f0 && f0 < s_pref[v + 1]) tstar = v;  // exactly one v matches
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) tstar = max(tstar, __shfl_xor_sync(0xffffffffu, tstar, m));
        long long run = s_pref[tstar];
        for (int base = tstar * per;; base += 32) {  // terminates inside thread tstar's chunk
            const int b = base + lane;
            long long n = 0;
            if (b < p.B && b < (tstar + 1) * per)
                n = (clamp_len(__ldg(p.seq_lens + b), p.W) + kBlockTokens - 1) / kBlockTokens;
            const long long incl = warp_incl_scan_ll(n * Y, lane) + run;
            const unsigned hit = __ballot_sync(0xffffffffu, incl > f0);
            if (hit) {
                const int src = __ffs(hit) - 1;
                cu.b = base + src;
                cu.seq_f = __shfl_sync(0xffffffffu, incl - n * Y, src);
                cu.nblk = static_cast<int>(__shfl_sync(0xffffffffu, n, src));
                break;
            }
            run = __shfl_sync(0xffffffffu, incl, 31);
        }
        cu.len = clamp_len(__ldg(p.seq_lens + cu.b), p.W);
        const long long off = f0 - cu.seq_f;
        cu.y = static_cast<int>(off / cu.nblk);
        cu.j = static_cast<int>(off % cu.nblk);
    }
    auto enter_segment = [&]() {
        const long long F0 = cu.seq_f + static_cast<long long>(cu.y) * cu.nblk;
        const long long F1 = F0 + cu.nblk;
        cu.seg_flags = (F0 >= f0 && F1 <= f1 ? kFlagWhole : 0) | (F0 >= f0 ? kFlagDir : 0);
        cu.w_hi = static_cast<int>((G * F1 - 1) / T);  // owner of tile F1 - 1
    };
    enter_segment();
    RowWindow win;
    win.reset(p.block_tables + static_cast<size_t>(cu.b) * p.W, cu.nblk, cu.j, lane);
    const uint64_t policy = l2_policy_evict_first();

    // Issues tile k (the cursor's position) into stage k % S and steps the cursor.
    auto issue = [&](int k) {
        const int32_t phys = win.get(cu.j);
        const int seg = cu.b * Y + cu.y;
        int flags = min(kBlockTokens, cu.len - cu.j * kBlockTokens) | cu.seg_flags;
        if (k == 0 || cu.j == 0) flags |= kFlagFirst;
        if (k == ntiles - 1 || cu.j == cu.nblk - 1) flags |= kFlagLast;
        const int w_hi = cu.w_hi;
        const bool ok = phys >= 0 && phys < p.num_blocks;
        const int s = k % S;
        if (lane == 0) {
            meta[s] = make_int4(ok ? phys : -1, seg, flags, w_hi);
            const uint32_t bar = bars + 8 * s;
            if (ok) {
                const uint32_t dst = smem_u32(ring + s * Geo::kStageBytes);
                const int yrow = phys * (p.Hkv * kBlockTokens) + (MMA ? cu.y / p.chunks : cu.y) * kBlockTokens;
                mbar_arrive_expect_tx(bar, Geo::kStageBytes);
#pragma unroll
                for (int hh = 0; hh < Geo::kHalves; ++hh) {
                    tma_load_2d(dst + hh * kBoxBytes, &tmk, hh * 64, yrow, bar, policy);
                    tma_load_2d(dst + Geo::kTileBytes + hh * kBoxBytes, &tmv, hh * 64, yrow, bar, policy);
                }
            } else {
                flag(p.err, PKV_DEV_ERR_BAD_BLOCK);
                mbar_arrive(bar);
            }
        }
        // step the cursor, unless this was the worker's last tile
        if (k + 1 >= ntiles) return;
        if (++cu.j < cu.nblk) {
            win.advance(cu.j, lane);
            return;
        }
        cu.j = 0;
        if (++cu.y == Y) {
            cu.y = 0;
            cu.seq_f += static_cast<long long>(cu.nblk) * Y;
            do {  // skip empty sequences; a later tile exists, so this ends before B
                ++cu.b;
                cu.len = clamp_len(__ldg(p.seq_lens + cu.b), p.W);
                cu.nblk = (cu.len + kBlockTokens - 1) / kBlockTokens;
            } while (cu.nblk == 0);
        }
        enter_segment();
        win.reset(p.block_tables + static_cast<size_t>(cu.b) * p.W, cu.nblk, 0, lane);
    };

    using Head = typename std::conditional<MMA, GroupHeads<D>, ScalarHead<D>>::type;
    Head st;
    for (int k = 0; k < S && k < ntiles; ++k) issue(k);

    int k = 0;
    for (; k < ntiles; ++k) {
        const int s = k % S;
        if (!mbar_wait(bars + 8 * s, static_cast<uint32_t>((k / S) & 1), kWaitLimitNs)) {
            if (lane == 0) flag(p.err, PKV_DEV_ERR_TIMEOUT);
            break;
        }
        const int4 m4 = meta[s];
        const int seg = m4.y, flags = m4.z;
        const int b = seg / Y, y = seg % Y;
        const int kvh = MMA ? y / p.chunks : y;
        const int h0 = MMA ? kvh * p.group + (y % p.chunks) * 8 : y;
        const int heads = MMA ? min(8, p.group - (y % p.chunks) * 8) : 1;
        const __nv_bfloat16 *qrow = p.q + (static_cast<size_t>(b) * p.Hq + h0) * D;
        if (flags & kFlagFirst) {
            if constexpr (MMA)
                st.init(qrow, heads, p.scale_log2, lane);
            else
                st.init(qrow, p.scale_log2, lane);
        }
        if (m4.x >= 0) {
            const uint8_t *kt = ring + s * Geo::kStageBytes;
            const int nvalid = flags & 0xFF;
            if constexpr (MMA)
                st.tile(smem_u32(kt), smem_u32(kt + Geo::kTileBytes), nvalid, lane);
            else
                st.tile(kt, kt + Geo::kTileBytes, nvalid, lane);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (k + S < ntiles) issue(k + S);

        if (flags & kFlagLast) {
            st.reduce();
            const size_t out_row = static_cast<size_t>(b) * p.Hq + h0;
            float *piece = p.ws_piece + static_cast<size_t>(w + seg) * p.HP * (D + 2);
            const bool whole = (flags & kFlagWhole) != 0;
            if constexpr (MMA) {
                const int tig = lane & 3, gid = lane >> 2;
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = 2 * tig + (i & 1);
                        const int d = 16 * mt + gid + (i >> 1) * 8;
                        if (n < heads) {
                            const float o = st.o[mt][i];
                            if (whole) {
                                const float l = st.l_run[i & 1];
                                p.out[(out_row + n) * D + d] = __float2bfloat16(l > 0.f ? o / l : 0.f);
                            } else {
                                piece[n * D + d] = o;
                            }
                        }
                    }
                if (!whole && gid == 0) {
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int n = 2 * tig + i;
                        if (n < heads) {
                            piece[p.HP * D + n] = st.m_run[i];
                            piece[p.HP * D + p.HP + n] = st.l_run[i];
                        }
                    }
                }
            } else {
                if (lane < Head::CH) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (whole)
                            p.out[out_row * D + st.c * 8 + e] =
                                __float2bfloat16(st.l_run > 0.f ? st.o[e] / st.l_run : 0.f);
                        else
                            piece[st.c * 8 + e] = st.o[e];
                    }
                }
                if (!whole && lane == 0) {
                    piece[D] = st.m_run;
                    piece[D + 1] = st.l_run;
                }
            }
            if ((flags & kFlagDir) && lane == 0)
                p.ws_dir[seg] = make_int2(static_cast<int>(w), m4.w);
        }
    }
    if (k < ntiles) {  // a wait gave up: let issued copies land before exiting (bounded)
        for (int j = k; j < ntiles && j < k + S; ++j)
            mbar_wait(bars + 8 * (j % S), static_cast<uint32_t>((j / S) & 1), kWaitLimitNs);
    }
}

// Log-sum-exp merge of the pieces of every segment cut by worker boundaries;
// writes the zero rows of empty sequences.  One CTA per segment, one thread
// per output column.
template <int D>
__global__ void __launch_bounds__(D) stream_merge_kernel(const StreamParams p) {
    const int seg = blockIdx.x, e = threadIdx.x;
    const int b = seg / p.Y, y = seg % p.Y;
    const int kvh = p.group > 1 ? y / p.chunks : y;
    const int h0 = p.group > 1 ? kvh * p.group + (y % p.chunks) * 8 : y;
    const int heads = p.group > 1 ? min(8, p.group - (y % p.chunks) * 8) : 1;
    const size_t out_row = static_cast<size_t>(b) * p.Hq + h0;
    if (clamp_len(__ldg(p.seq_lens + b), p.W) == 0) {
        for (int n = 0; n < heads; ++n) p.out[(out_row + n) * D + e] = __float2bfloat16(0.f);
        return;
    }
    const int2 dir = p.ws_dir[seg];
    if (dir.x == dir.y) return;  // finished by its only worker
    // With fewer tiles than workers some workers own no tile; they left no piece.
    const long long T = *p.ws_total, G = p.num_workers;
    const auto has_tiles = [&](int w) { return (w + 1) * T / G > w * T / G; };
    for (int n = 0; n < heads; ++n) {
        float M = -INFINITY;
        for (int w = dir.x; w <= dir.y; ++w) {
            if (!has_tiles(w)) continue;
            const float *pc = p.ws_piece + static_cast<size_t>(w + seg) * p.HP * (D + 2);
            M = fmaxf(M, pc[p.HP * D + n]);
        }
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
            for (int w = dir.x; w <= dir.y; ++w) {
                if (!has_tiles(w)) continue;
                const float *pc = p.ws_piece + static_cast<size_t>(w + seg) * p.HP * (D + 2);
                const float c = exp2f(pc[p.HP * D + n] - M);
                L = fmaf(pc[p.HP * D + p.HP + n], c, L);
                O = fmaf(pc[n * D + e], c, O);
            }
        }
        p.out[(out_row + n) * D + e] = __float2bfloat16(L > 0.f ? O / L : 0.f);
    }
}

template <int D, int NW, int S, bool MMA>
cudaError_t launch_stream_one(const CUtensorMap &tmk, const CUtensorMap &tmv, StreamParams p,
                              cudaStream_t stream) {
    using Geo = Geometry<D, NW, S>;
    constexpr int kSmem = Geo::kSmemBytes + NW * S * 16 + (NW * 32 + 1) * 8;
    auto kern = paged_decode_stream_kernel<D, NW, S, MMA>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NW * 32, kSmem)) != cudaSuccess)
        return e;
    per_sm = max(1, min(per_sm, kStreamMaxCtasPerSm));
    const int grid = sms * per_sm;
    if (static_cast<long long>(grid) * NW > p.max_workers) return cudaErrorInvalidValue;
    p.num_workers = static_cast<long long>(grid) * NW;
    kern<<<grid, NW * 32, kSmem, stream>>>(tmk, tmv, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stream_merge_kernel<D><<<p.B * p.Y, D, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_stream(const CUtensorMap &tmk, const CUtensorMap &tmv,
                                 const StreamParams &p, int head_dim, cudaStream_t stream) {
    const bool mma = p.group > 1;
    if (head_dim == 128)
        return mma ? launch_stream_one<128, 4, 2, true>(tmk, tmv, p, stream)
                   : launch_stream_one<128, 4, 2, false>(tmk, tmv, p, stream);
    if (head_dim == 64)
        return mma ? launch_stream_one<64, 4, 2, true>(tmk, tmv, p, stream)
                   : launch_stream_one<64, 4, 2, false>(tmk, tmv, p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pkv
