// Paged prefill attention on the 5th-generation tensor cores (tcgen05, TMEM).
//
// Causal attention of each sequence's new tokens over its paged K/V ("vLLM 與
// PagedAttention：高吞吐推理的關鍵", section 三 step 二).  A persistent CTA (one per SM) walks work
// items; an item is two Q tiles of 128 query rows each -- (token, query head
// of one KV head) pairs of one sequence -- whose keys are walked in tiles of
// 128 (eight 16-token blocks); both Q tiles share each K/V tile.  Per Q tile x:
//   S_x[128 x 128] = Q_x[128 x d] K_tile^T   tcgen05.mma (A, B in shared memory)
//   P_x = exp2(S_x - m), bf16, written back into TMEM over S_x
//   O_x[128 x d]  += P_x V_tile              tcgen05.mma (A in TMEM, B in shared memory)
// with S, P and O accumulated in TMEM (512 columns).
// Roles: a producer warp streams K and V tiles (TMA, 128-byte swizzle, K and
// V in separate rings; blocks past the table or the pool load as zeros from
// out-of-range coordinates); one thread of the MMA warp issues the products
// and commits them to mbarriers; one softmax warpgroup per Q tile owns one
// row per thread (TMEM lane = row), reads S with tcgen05.ld, masks (causal,
// sequence end), keeps the running max and sum, stores P with tcgen05.st, and
// rescales O in TMEM only when a row's max grows by more than 2^8 (otherwise
// the old max is kept: P stays <= 2^8).  The two Q tiles ping-pong: the tensor
// core computes one tile's products while the other tile's softmax runs.
// Every wait is bounded; on a timeout the kernel flags PKV_DEV_ERR_TIMEOUT,
// stops issuing, and still frees its TMEM.
#include <algorithm>

#include "decode_common.cuh"
#include "tcgen05.cuh"

namespace pkv {

namespace {

using namespace dev;

constexpr int kRows = 128;                 // query rows per Q tile (MMA M)
constexpr int kTiles = 2;                  // Q tiles per CTA, ping-ponged on the tensor core
constexpr int kCtaRows = kTiles * kRows;
constexpr int kKeys = 128;                 // keys per tile (MMA N of S, K of P.V)
constexpr int kWarpsPerTile = 4;           // one softmax warpgroup per Q tile
constexpr int kSoftmaxWarps = kTiles * kWarpsPerTile;
constexpr int kProducerWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
constexpr int kQWarp = kSoftmaxWarps + 2;  // + x: the Q rows of tile x
constexpr int kThreads = (kSoftmaxWarps + 2 + kTiles) * 32;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// ------------------------------------------------ packed f32x2 arithmetic
// Two floats in one 64-bit register pair for the sm_100 f32x2 instructions.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int D>
struct TcGeometry {
    static constexpr int kHalves = D / 64;
    static constexpr int kKStages = D == 128 ? 3 : 4;           // K ring depth
    static constexpr int kVStages = D == 128 ? 2 : 4;           // V ring depth
    static constexpr int kQBytes = kHalves * kRows * 128;      // one Q tile [half][row][128 B]
    static constexpr int kKVBytes = kHalves * kKeys * 128;     // K or V tile [half][key][128 B]
    static constexpr int kQ = 0;                               // + tile * kQBytes
    static constexpr int kK = kQ + kTiles * kQBytes;           // + stage * kKVBytes
    static constexpr int kV = kK + kKStages * kKVBytes;
    static constexpr int kBars = kV + kVStages * kKVBytes;     // up to 32 mbarriers
    static constexpr int kTmemSlot = kBars + 32 * 8;
    static constexpr int kSmemBytes = kTmemSlot + 16 + 1024;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
    static_assert(2 * (kKStages + kVStages) + 12 <= 32, "barrier slots");
    // TMEM columns: S of tile x at kKeys x (P, bf16, over its first half),
    // O of tile x at kO + D x.
    static constexpr int kO = kTiles * kKeys;
    static constexpr int kTmemCols = 512;
    static_assert(kO + kTiles * D <= kTmemCols, "tensor memory columns");
};

// One work item: 256 query rows (two Q tiles) of one (sequence, KV head).
struct TcItem {
    int b, kvh, q0, ctx, rows, r_begin, first_pos, nblk_seq;
    int nk0, nk1;  // key tiles Q tile 0 / 1 can see (tile 1 may be empty: 0)
};

// Items are numbered z-major -- z counts 256-row tiles from the END of each
// sequence, so low numbers see the most keys -- then sequence, then KV head.
// Returns false for items past a sequence's rows or of a sequence whose
// lengths are inconsistent (*bad set for the latter).
__device__ __forceinline__ bool tc_item(const PrefillParams &p, int i, TcItem &it, bool *bad) {
    const int per_z = p.Hkv * p.B;
    const int z = i / per_z, rem = i - z * per_z;
    it.b = rem / p.Hkv;
    it.kvh = rem - it.b * p.Hkv;
    it.q0 = __ldg(p.query_start + it.b);
    const int nq = __ldg(p.query_start + it.b + 1) - it.q0;
    it.ctx = __ldg(p.seq_lens + it.b);
    *bad = nq > 0 && (it.ctx < nq || it.ctx > p.W * kBlockTokens);
    if (nq <= 0 || *bad) return false;
    it.rows = nq * p.group;
    const int ntile = (it.rows + kCtaRows - 1) / kCtaRows;
    if (z >= ntile) return false;
    it.r_begin = (ntile - 1 - z) * kCtaRows;
    it.first_pos = it.ctx - nq;
    it.nblk_seq = (it.ctx + kBlockTokens - 1) / kBlockTokens;
    const int last0 = min(it.rows, it.r_begin + kRows) - 1;
    it.nk0 = (it.first_pos + last0 / p.group + kKeys) / kKeys;
    const int lo1 = it.r_begin + kRows;
    it.nk1 = lo1 < it.rows ? (it.first_pos + (min(it.rows, lo1 + kRows) - 1) / p.group + kKeys) / kKeys : 0;
    return true;
}

// The k-th item of CTA c in a grid of n CTAs: rounds of n items, alternately
// forwards and backwards ("snake"), so heavy and light items even out.
__device__ __forceinline__ int tc_item_index(int k, int c, int n) {
    return k * n + ((k & 1) ? n - 1 - c : c);
}

// Next valid item of this CTA at or after round k; returns its round or -1.
__device__ __forceinline__ int tc_next_item(const PrefillParams &p, int k, TcItem &it) {
    for (;; ++k) {
        const int i = tc_item_index(k, blockIdx.x, gridDim.x);
        if (i >= p.items) return -1;
        bool bad;
        if (tc_item(p, i, it, &bad)) return k;
    }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

// Persistent: one CTA per SM walks its items; TMEM is allocated once, every
// barrier's phase runs on across items, and a dedicated warp fetches the next
// item's Q rows (cp.async) as soon as the current item's last S product of
// that Q tile is done.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv, const PrefillParams p) {
    using Geo = TcGeometry<D>;
    constexpr int KS = Geo::kKStages, VS = Geo::kVStages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t bar0 = smem_u32(smem + Geo::kBars);
    // barriers: k_full[KS] k_empty[KS] v_full[VS] v_empty[VS], then per Q tile
    // s_full p_full o_done q_full o_free q_free
    const auto k_full = [&](int s) { return bar0 + 8 * s; };
    const auto k_empty = [&](int s) { return bar0 + 8 * (KS + s); };
    const auto v_full = [&](int s) { return bar0 + 8 * (2 * KS + s); };
    const auto v_empty = [&](int s) { return bar0 + 8 * (2 * KS + VS + s); };
    const uint32_t tile_bars = bar0 + 8 * (2 * KS + 2 * VS);
    const auto s_full = [&](int x) { return tile_bars + 8 * x; };
    const auto p_full = [&](int x) { return tile_bars + 8 * (2 + x); };
    const auto o_done = [&](int x) { return tile_bars + 8 * (4 + x); };
    const auto q_full = [&](int x) { return tile_bars + 8 * (6 + x); };
    const auto o_free = [&](int x) { return tile_bars + 8 * (8 + x); };
    const auto q_free = [&](int x) { return tile_bars + 8 * (10 + x); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Geo::kTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Geo::kTmemSlot + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < KS; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(k_empty(s), 1);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(v_full(s), 1);
            mbar_init(v_empty(s), 1);
        }
        for (int x = 0; x < kTiles; ++x) {
            mbar_init(s_full(x), 1);
            mbar_init(p_full(x), kWarpsPerTile);
            mbar_init(o_done(x), 1);
            mbar_init(q_full(x), 1);
            mbar_init(o_free(x), kWarpsPerTile);
            mbar_init(q_free(x), 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    if (warp == kMmaWarp) {
        tc::alloc<Geo::kTmemCols>(smem_u32(tmem_slot));
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kProducerWarp) {
        if (lane == 0) {
            const uint64_t policy = l2_policy_evict_normal();
            int gk = 0, gv = 0;  // K / V tiles loaded so far (ring position and phase)
            TcItem it, nx;
            for (int k = tc_next_item(p, 0, it); k >= 0 && !*abort_flag; it = nx) {
                const int kn = tc_next_item(p, k + 1, nx);
                const int32_t *trow = p.block_tables + static_cast<size_t>(it.b) * p.W;
                const int nk = max(it.nk0, it.nk1);
                for (int j = 0; j < nk && !*abort_flag; ++j) {
                    int y[kKeys / kBlockTokens];  // tensor-map rows of the tile's blocks
#pragma unroll
                    for (int i = 0; i < kKeys / kBlockTokens; ++i) {
                        const int blk = j * (kKeys / kBlockTokens) + i;
                        long long yy = p.num_blocks * p.Hkv * kBlockTokens;  // past the tensor: zeros
                        if (blk < it.nblk_seq) {
                            const int32_t phys = __ldg(trow + blk);
                            if (phys >= 0 && phys < p.num_blocks)
                                yy = (static_cast<long long>(phys) * p.Hkv + it.kvh) * kBlockTokens;
                            else
                                flag(p.err, PKV_DEV_ERR_BAD_BLOCK);
                        }
                        y[i] = static_cast<int>(yy);
                    }
                    const int sk = gk % KS, sv = gv % VS;
                    if (gk >= KS &&
                        !mbar_wait(k_empty(sk), static_cast<uint32_t>((gk / KS - 1) & 1), kWaitLimitNs)) {
                        flag(p.err, PKV_DEV_ERR_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(k_full(sk), Geo::kKVBytes);
#pragma unroll
                    for (int i = 0; i < kKeys / kBlockTokens; ++i)
#pragma unroll
                        for (int hh = 0; hh < Geo::kHalves; ++hh)
                            tma_load_2d(smem_u32(smem + Geo::kK + sk * Geo::kKVBytes) +
                                            hh * (kKeys * 128) + i * (kBlockTokens * 128),
                                        &tmk, hh * 64, y[i], k_full(sk), policy);
                    ++gk;
                    if (gv >= VS &&
                        !mbar_wait(v_empty(sv), static_cast<uint32_t>((gv / VS - 1) & 1), kWaitLimitNs)) {
                        flag(p.err, PKV_DEV_ERR_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(v_full(sv), Geo::kKVBytes);
#pragma unroll
                    for (int i = 0; i < kKeys / kBlockTokens; ++i)
#pragma unroll
                        for (int hh = 0; hh < Geo::kHalves; ++hh)
                            tma_load_2d(smem_u32(smem + Geo::kV + sv * Geo::kKVBytes) +
                                            hh * (kKeys * 128) + i * (kBlockTokens * 128),
                                        &tmv, hh * 64, y[i], v_full(sv), policy);
                    ++gv;
                }
                k = kn;
            }
            // on an abort, copies may still be landing: wait (bounded) for the last of each stage
            for (int g = max(gk - KS, 0); g < gk; ++g)
                mbar_wait(k_full(g % KS), static_cast<uint32_t>((g / KS) & 1), kWaitLimitNs);
            for (int g = max(gv - VS, 0); g < gv; ++g)
                mbar_wait(v_full(g % VS), static_cast<uint32_t>((g / VS) & 1), kWaitLimitNs);
            // sequences whose lengths do not fit: flagged once each (item z = 0, KV head 0)
            for (int k = 0;; ++k) {
                const int i = tc_item_index(k, blockIdx.x, gridDim.x);
                if (i >= p.items) break;
                if (i < p.Hkv * p.B && i % p.Hkv == 0) {
                    TcItem bad_it;
                    bool bad;
                    tc_item(p, i, bad_it, &bad);
                    if (bad) flag(p.err, PKV_DEV_ERR_BAD_LEN);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // Per item: S_0(0), S_1(0); then per key tile j: PV_0(j), S_0(j+1),
        // PV_1(j), S_1(j+1).  The tensor core runs them in that order, so
        // while tile 0's softmax works on S_0(j+1) the products of tile 1
        // proceed, and the other way round.  S_x(j+1) is issued only after
        // P_x(j) is ready, by which time tile x's softmax has read S_x(j) out
        // of TMEM; it overwrites P_x(j) (which aliases S_x) only after PV_x(j),
        // issued before it, has read it; and its completion tells the
        // softmax that PV_x(j) is done.
        constexpr uint32_t kIdS = tc::idesc_bf16(kRows, kKeys, 0);
        constexpr uint32_t kIdO = tc::idesc_bf16(kRows, D, 1);
        const auto issue_s = [&](int x, int stage) {  // S_x = Q_x . K^T
            const uint32_t kbase = smem_u32(smem + Geo::kK + stage * Geo::kKVBytes);
            const uint32_t qbase = smem_u32(smem + Geo::kQ + x * Geo::kQBytes);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const int hh = k >> 2, kk = k & 3;
                tc::mma_ss(tmem + kKeys * x, tc::smem_desc(qbase + hh * (kRows * 128) + kk * 32, 16, 1024),
                     tc::smem_desc(kbase + hh * (kKeys * 128) + kk * 32, 16, 1024), kIdS, k > 0);
            }
            tc::commit(s_full(x));
        };
        const auto issue_pv = [&](int x, int stage, bool acc) {  // O_x (+)= P_x . V, P_x from TMEM
            const uint32_t vbase = smem_u32(smem + Geo::kV + stage * Geo::kKVBytes);
#pragma unroll
            for (int k = 0; k < kKeys / 16; ++k)
                tc::mma_ts(tmem + Geo::kO + D * x, tmem + kKeys * x + 8 * k,
                        tc::smem_desc(vbase + k * (16 * 128), kKeys * 128, 1024), kIdO, acc || k > 0);
        };
        bool ok = true;
        const auto wait = [&](uint32_t bar, uint32_t parity) {
            if (!ok) return;
            if (!mbar_wait(bar, parity, kWaitLimitNs) || *abort_flag) {
                ok = false;
                if (lane == 0) {
                    flag(p.err, PKV_DEV_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
            }
        };
        int gk = 0, gv = 0;      // K / V tiles consumed
        int ns[kTiles] = {0, 0};  // S products per Q tile (s_full / p_full phases)
        int n_it = 0;            // items done (q_full / o_done / o_free phases)
        TcItem it, nx;
        int k = tc_next_item(p, 0, it);
        for (; k >= 0 && ok; it = nx, ++n_it) {
            // the next item's parameters are read now, off the item boundary
            const int kn = tc_next_item(p, k + 1, nx);
            const int nk_t[kTiles] = {it.nk0, it.nk1};
            const int nk = max(it.nk0, it.nk1);
            wait(k_full(gk % KS), static_cast<uint32_t>((gk / KS) & 1));
#pragma unroll
            for (int x = 0; x < kTiles; ++x) {
                if (nk_t[x] == 0) continue;
                wait(q_full(x), static_cast<uint32_t>(n_it & 1));
                tc::fence_after();
                if (ok && lane == 0) {
                    issue_s(x, gk % KS);
                    if (nk_t[x] == 1) tc::commit(q_free(x));  // the item's last S_x has read Q_x
                }
                __syncwarp();
            }
            if (ok && lane == 0) tc::commit(k_empty(gk % KS));
            __syncwarp();
            ++gk;
            for (int j = 0; j < nk && ok; ++j, ++gv) {
                const int sv = gv % VS;
                wait(v_full(sv), static_cast<uint32_t>((gv / VS) & 1));
                // V rows of slots at or past the sequence end may hold anything: zero them
                const int k_lo = j * kKeys;
                if (ok && k_lo + kKeys > it.ctx && k_lo < it.nblk_seq * kBlockTokens) {
                    const int z0 = max(it.ctx - k_lo, 0), z1 = min(it.nblk_seq * kBlockTokens - k_lo, kKeys);
                    uint8_t *vbase = smem + Geo::kV + sv * Geo::kKVBytes;
                    for (int idx = lane; idx < (z1 - z0) * Geo::kHalves * 8; idx += 32) {
                        const int rr = z0 + idx / (Geo::kHalves * 8), rest = idx % (Geo::kHalves * 8);
                        *reinterpret_cast<uint4 *>(vbase + (rest >> 3) * (kKeys * 128) + rr * 128 +
                                                   ((rest & 7) << 4)) = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                // the last tile that reads V_j (and K_{j+1}) releases its stage
                const int last_v = j < nk_t[1] ? 1 : 0;
                const int last_k = j + 1 < nk_t[1] ? 1 : 0;
                bool next_ready = false;
#pragma unroll
                for (int x = 0; x < kTiles; ++x) {
                    if (j >= nk_t[x]) continue;
                    wait(p_full(x), static_cast<uint32_t>(ns[x] & 1));
                    if (j == 0 && n_it > 0) wait(o_free(x), static_cast<uint32_t>((n_it - 1) & 1));
                    tc::fence_after();
                    if (ok && lane == 0) {
                        issue_pv(x, sv, j > 0);
                        if (x == last_v) tc::commit(v_empty(sv));
                        if (j + 1 >= nk_t[x]) tc::commit(o_done(x));
                    }
                    ++ns[x];
                    if (j + 1 < nk_t[x]) {
                        if (!next_ready) {
                            wait(k_full(gk % KS), static_cast<uint32_t>((gk / KS) & 1));
                            tc::fence_after();
                            next_ready = true;
                        }
                        if (ok && lane == 0) {
                            issue_s(x, gk % KS);
                            if (x == last_k) tc::commit(k_empty(gk % KS));
                            if (j + 2 == nk_t[x]) tc::commit(q_free(x));  // the item's last S_x
                        }
                    }
                    __syncwarp();
                }
                if (next_ready) ++gk;
            }
            // a Q tile without rows in this item still takes its phases
            for (int x = 0; x < kTiles; ++x) {
                if (nk_t[x] > 0) continue;
                wait(q_full(x), static_cast<uint32_t>(n_it & 1));
                if (n_it > 0) wait(o_free(x), static_cast<uint32_t>((n_it - 1) & 1));
                if (ok && lane == 0) {
                    tc::commit(o_done(x));
                    tc::commit(q_free(x));
                }
                __syncwarp();
            }
            k = kn;
        }
    } else if (warp >= kQWarp) {
        // ---------------- Q rows of each item into shared memory (K-major,
        // 128-byte swizzle; rows past the item's rows zero-filled), one warp
        // per Q tile: tile x's rows of item n once the last S_x product of
        // item n - 1 has read Q_x (q_free), then q_full.  Off the softmax
        // warps, whose last step of an item this 32 KB of cp.async per tile
        // used to lengthen.
        const int x = warp - kQWarp;
        bool ok = true;
        int n_it = 0;
        TcItem it, nx;
        for (int k = tc_next_item(p, 0, it); k >= 0 && ok; it = nx, ++n_it) {
            const int kn = tc_next_item(p, k + 1, nx);
            {
                if (n_it > 0 && (!mbar_wait(q_free(x), static_cast<uint32_t>((n_it - 1) & 1), kWaitLimitNs) ||
                                 *abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t *qtile = smem + Geo::kQ + x * Geo::kQBytes;
#pragma unroll 1
                for (int rr = lane; rr < kRows; rr += 32) {
                    const int r = it.r_begin + x * kRows + rr;
                    const __nv_bfloat16 *src = p.q;
                    uint32_t bytes = 0;
                    if (r < it.rows) {
                        src = p.q + (static_cast<size_t>(it.q0 + r / G) * p.Hq + it.kvh * G + r % G) * D;
                        bytes = 16;
                    }
#pragma unroll
                    for (int c = 0; c < D / 8; ++c)
                        cp_async16(smem_u32(qtile + (c >> 3) * (kRows * 128) + rr * 128 + (((c & 7) ^ (rr & 7)) << 4)),
                                   src + (bytes ? c * 8 : 0), bytes);
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
                asm volatile("cp.async.wait_all;" ::: "memory");
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(q_full(x));
            }
            k = kn;
        }
        if (!ok && lane == 0) {
            flag(p.err, PKV_DEV_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else {
        // ---------------- softmax warps: thread t of tile x = TMEM lane t = row r_begin + 128 x + t
        const int tile = warp / kWarpsPerTile;
        const int t = threadIdx.x & (kRows - 1);
        const uint32_t lane_addr = static_cast<uint32_t>((warp % kWarpsPerTile) * 32) << 16;
        const uint32_t t_s = tmem + lane_addr + kKeys * tile;
        const uint32_t t_o = tmem + lane_addr + Geo::kO + D * tile;
        bool ok = true;
        int ns = 0;    // S products seen (s_full / p_full phases)
        int n_it = 0;  // items done (o_done phases)
        TcItem it, nx;  // the current and the next item
        int k = tc_next_item(p, 0, it);
        while (k >= 0 && ok) {
            const int kn = tc_next_item(p, k + 1, nx);
            const int r = it.r_begin + tile * kRows + t;
            const int row_pos = r < it.rows ? it.first_pos + r / G : -1;
            const int my_nk = tile == 0 ? it.nk0 : it.nk1;
            __nv_bfloat16 *out_row =
                p.out + (static_cast<size_t>(it.q0 + r / G) * p.Hq + it.kvh * G + r % G) * D;
            float m_run = -INFINITY, l_run = 0.f;
            for (int j = 0; j < my_nk; ++j, ++ns) {
                // S_x(j) done; it was issued after PV_x(j - 1), so O_x is free too
                if (!mbar_wait(s_full(tile), static_cast<uint32_t>(ns & 1), kWaitLimitNs) || *abort_flag) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                // Two passes over S in TMEM, 64 columns at a time, so that a row
                // never sits in registers whole (twelve warps leave 170 registers
                // a thread): the row max first, then exp2 and P.
                const int k0 = j * kKeys;
                const bool masked = __any_sync(0xffffffffu, k0 + kKeys - 1 > row_pos);
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1  // one half's 64 registers live at a time
                for (int h = 0; h < kKeys / 64; ++h) {
                    // causal mask by position (only tiles that reach past some row
                    // need it), decided per 64-key half and warp: a half past
                    // every row of the warp is skipped, one before every row
                    // needs no mask
                    const int lim = row_pos - (k0 + 64 * h);  // keys c > lim are masked
                    if (masked && __all_sync(0xffffffffu, lim < 0)) continue;
                    uint32_t sr[64];
                    tc::ld32(t_s + 64 * h, sr);
                    tc::ld32(t_s + 64 * h + 32, sr + 32);
                    tc::wait_ld();
                    if (masked && !__all_sync(0xffffffffu, lim >= 63)) {
#pragma unroll
                        for (int c = 0; c < 64; ++c)
                            if (c > lim) sr[c] = 0xFF800000u;  // -inf
                    }
#pragma unroll
                    for (int c = 0; c < 64; c += 2)
                        mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
                }
                // row max of the raw scores (scale > 0)
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * p.scale_log2;
                // keep the running max unless it grows by more than 2^8
                const bool grow = mx > m_run + kRescaleThreshold || (m_run == -INFINITY && mx != -INFINITY);
                const float m_new = grow ? mx : m_run;
                const float nbase = m_new == -INFINITY ? 0.f : -m_new;
                // P_x over the first half of S_x's columns (two keys per column),
                // 64 keys at a time; P's columns [32 h, 32 h + 32) overwrite S
                // columns already read
                const uint64_t scale2 = f2pack(p.scale_log2, p.scale_log2);
                const uint64_t nbase2 = f2pack(nbase, nbase);
                uint64_t sum2[2] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
#pragma unroll 1  // one half's 64 registers live at a time
                for (int h = 0; h < kKeys / 64; ++h) {
                    const int lim = row_pos - (k0 + 64 * h);
                    uint32_t pk[32];
                    if (masked && __all_sync(0xffffffffu, lim < 0)) {  // P = 0 over the whole half
#pragma unroll
                        for (int c = 0; c < 32; ++c) pk[c] = 0u;
                        tc::st32(t_s + 32 * h, pk);
                        continue;
                    }
                    uint32_t sr[64];
                    tc::ld32(t_s + 64 * h, sr);
                    tc::ld32(t_s + 64 * h + 32, sr + 32);
                    tc::wait_ld();
                    if (masked && !__all_sync(0xffffffffu, lim >= 63)) {  // -inf scores (2^-inf = 0)
#pragma unroll
                        for (int c = 0; c < 64; ++c)
                            if (c > lim) sr[c] = 0xFF800000u;
                    }
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {  // scale and shift two at a time, 2^x on the SFU
                        float a, bb;
                        f2unpack(ffma2(f2pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), scale2, nbase2), a, bb);
                        a = ex2_approx(a);
                        bb = ex2_approx(bb);
                        sum2[(c >> 1) & 1] = fadd2(sum2[(c >> 1) & 1], f2pack(a, bb));
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(a, bb);
                        pk[c / 2] = *reinterpret_cast<uint32_t *>(&h2);
                    }
                    tc::st32(t_s + 32 * h, pk);
                }
                float s_lo, s_hi, s_lo2, s_hi2;
                f2unpack(sum2[0], s_lo, s_hi);
                f2unpack(sum2[1], s_lo2, s_hi2);
                const float rowsum = (s_lo + s_hi) + (s_lo2 + s_hi2);
                if (j > 0) {
                    const float alpha = (grow && m_run != -INFINITY) ? exp2f(m_run - m_new) : 1.f;
                    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                        for (int cc = 0; cc < D / 32; ++cc) {
                            uint32_t o[32];
                            tc::ld32(t_o + 32 * cc, o);
                            tc::wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                            tc::st32(t_o + 32 * cc, o);
                        }
                    }
                    l_run *= alpha;
                }
                l_run += rowsum;
                m_run = m_new;
                tc::wait_st();
                tc::fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full(tile));
            }
            if (!ok) break;
            // O_x of this item complete (a tile without rows gets a bare commit)
            if (!mbar_wait(o_done(tile), static_cast<uint32_t>(n_it & 1), kWaitLimitNs) || *abort_flag) {
                ok = false;
                break;
            }
            tc::fence_after();
            ++n_it;
            if (my_nk == 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(o_free(tile));
                it = nx;
                k = kn;
                continue;
            }
            // O row, normalised, packed to bf16 and stored 64 columns at a
            // time; then O_x is handed back
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            uint4 *dst = reinterpret_cast<uint4 *>(out_row);
#pragma unroll
            for (int h = 0; h < D / 64; ++h) {
                uint32_t o[64];
                tc::ld32(t_o + 64 * h, o);
                tc::ld32(t_o + 64 * h + 32, o + 32);
                tc::wait_ld();
                if (row_pos >= 0) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[8 * i + 2 * e]) * inv,
                                                                      __uint_as_float(o[8 * i + 2 * e + 1]) * inv);
                            w[e] = *reinterpret_cast<uint32_t *>(&h2);
                        }
                        dst[8 * h + i] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free(tile));
            it = nx;
            k = kn;
        }
        if (!ok && t == 0) {
            flag(p.err, PKV_DEV_ERR_TIMEOUT);
            *abort_flag = 1;
        }
    }
    // everyone (the producer's copies included) is done with TMEM and shared memory
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == kMmaWarp)
        tc::dealloc<Geo::kTmemCols>(tmem);
}

template <int D>
cudaError_t launch_prefill_tc_d(const CUtensorMap &tmk, const CUtensorMap &tmv, PrefillParams p,
                                int max_query_len, int num_sms, cudaStream_t stream) {
    constexpr int kSmem = TcGeometry<D>::kSmemBytes;
    auto kern = paged_prefill_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    const long long rows = static_cast<long long>(max_query_len) * p.group;
    const long long items = (rows + kCtaRows - 1) / kCtaRows * p.Hkv * p.B;
    if (items == 0) return cudaSuccess;
    if (items > 0x7FFFFFFFLL - 2LL * num_sms) return cudaErrorInvalidValue;
    p.items = static_cast<int>(items);
    const unsigned grid = static_cast<unsigned>(std::min<long long>(items, num_sms));
    kern<<<grid, kThreads, kSmem, stream>>>(tmk, tmv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefillParams &p,
                              int head_dim, int max_query_len, int num_sms, cudaStream_t stream) {
    if (head_dim == 128) return launch_prefill_tc_d<128>(tmk, tmv, p, max_query_len, num_sms, stream);
    if (head_dim == 64) return launch_prefill_tc_d<64>(tmk, tmv, p, max_query_len, num_sms, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pkv
