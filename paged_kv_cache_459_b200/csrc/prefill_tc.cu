// Paged prefill attention on the 5th-generation tensor cores (tcgen05, TMEM).
//
// Causal attention of each sequence's new tokens over its paged K/V ("vLLM 與
// PagedAttention：高吞吐推理的關鍵", section 三 step 二).  A persistent CTA (one per
// SM) walks work items; an item is two Q tiles of 128 query rows each -- (token, query head
// of one KV head) pairs of one sequence -- whose keys are walked in tiles of
// 128 (eight 16-token blocks); both Q tiles share each K/V tile.  Per Q tile x:
//   S_x[128 x 128] = Q_x[128 x d] K_tile^T   tcgen05.mma (A, B in shared memory)
//   P_x = exp2(S_x - m), bf16, written back into TMEM over S_x
//   O_x[128 x d]  += P_x V_tile              tcgen05.mma (A in TMEM, B in shared memory)
// with S, P and O accumulated in TMEM (512 columns).
// Roles: a producer warp streams K and V tiles (TMA, 128-byte swizzle, K and
// V in separate rings; blocks past the table or the pool load as zeros from
// out-of-range coordinates); one thread of the MMA warp issues the products
// and commits them to mbarriers; two softmax warpgroups per Q tile each own
// half of every key tile (64 keys) for one row per thread (TMEM lane = row):
// they read S with tcgen05.ld, mask (causal, sequence end), trade their row
// maxima through shared memory behind the tile's named barrier, keep the
// running max and sum, store P with tcgen05.st, and rescale their half of O
// in TMEM only when a row's max grows by more than 2^8 (otherwise the old max
// is kept: P stays <= 2^8).  Halving each tile's softmax shortens its chain
// S -> softmax -> P.V -> next S, which bounds the step.  The two Q tiles
// ping-pong: the tensor core computes one tile's products while the other
// tile's softmax runs.  Every mbarrier wait is bounded; a wait that gives up
// is voted on at the tile's next named barrier so that all its warps stop
// together; the kernel flags PKV_DEV_ERR_TIMEOUT, stops issuing, and still
// frees its TMEM.
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
constexpr int kWarpsPerTile = 4;           // warps of one softmax warpgroup (all 128 TMEM lanes)
constexpr int kSoftmaxWarps = kTiles * 2 * kWarpsPerTile;  // two warpgroups (key halves) per Q tile
constexpr int kProducerWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
constexpr int kThreads = (kSoftmaxWarps + 2) * 32;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Of every 16 score pairs a softmax thread turns into P, this many take 2^x
// on the FMA pipe (exp2_fma2) instead of the special-function unit, which
// the two Q tiles' softmaxes otherwise share.
constexpr int kFmaExpPairs = 0;

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
__device__ __forceinline__ uint64_t fsub2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x for two values on the FMA pipe instead of the special-function unit:
// 2^x = 2^floor(x) * 2^f, f in [0, 1), with 2^f from a cubic fitted here to
// 2^f on [0, 1) by least squares on the relative error (largest relative
// error 2.2e-4, under the bf16 rounding of P); the integer part is added to
// the exponent bits.  x is clamped at -126 (2^-126 instead of 0 below it);
// the softmax never passes more than +8.
__device__ __forceinline__ void exp2_fma2(float &a, float &b) {
    constexpr float c0 = 0.99998891353607178f, c1 = 0.69449967145919800f;
    constexpr float c2 = 0.23030571639537811f, c3 = 0.07476584613323212f;
    a = fmaxf(a, -126.f);
    b = fmaxf(b, -126.f);
    const float fa = floorf(a), fb = floorf(b);
    const uint64_t f = fsub2(f2pack(a, b), f2pack(fa, fb));
    uint64_t p = ffma2(f2pack(c3, c3), f, f2pack(c2, c2));
    p = ffma2(p, f, f2pack(c1, c1));
    p = ffma2(p, f, f2pack(c0, c0));
    float pa, pb;
    f2unpack(p, pa, pb);
    a = __uint_as_float(__float_as_uint(pa) + (static_cast<uint32_t>(static_cast<int>(fa)) << 23));
    b = __uint_as_float(__float_as_uint(pb) + (static_cast<uint32_t>(static_cast<int>(fb)) << 23));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int D>
struct TcGeometry {
    static constexpr int kHalves = D / 64;
    static constexpr int kKStages = D == 128 ? 2 : 4;           // K ring depth
    static constexpr int kVStages = D == 128 ? 2 : 4;           // V ring depth
    static constexpr int kQBytes = kHalves * kRows * 128;      // one Q tile [half][row][128 B]
    static constexpr int kKVBytes = kHalves * kKeys * 128;     // K or V tile [half][key][128 B]
    static constexpr int kQ = 0;                               // + tile * kQBytes
    static constexpr int kK = kQ + kTiles * kQBytes;           // + stage * kKVBytes
    static constexpr int kV = kK + kKStages * kKVBytes;
    static constexpr int kBars = kV + kVStages * kKVBytes;     // up to 32 mbarriers
    static constexpr int kTmemSlot = kBars + 32 * 8;
    // per Q tile: the key halves' row maxima and row sums (2 parities each)
    // and the warps' votes (2 step parities, 2 item parities, 8 warps each)
    static constexpr int kXchPerTile = 8 * kRows + 32;        // floats
    static constexpr int kXch = kTmemSlot + 16;
    static constexpr int kSmemBytes = kXch + kTiles * kXchPerTile * 4 + 1024;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
    static_assert(2 * (kKStages + kVStages) + 10 <= 32, "barrier slots");
    // TMEM columns: S of tile x at kKeys x (P, bf16, over columns [0, 32) and
    // [64, 96) of it: each softmax half's keys over its own scores),
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

// z counts 256-row tiles from the END of each sequence, so low z sees the
// most keys.  Items are numbered heaviest first in groups of kZGroup z levels:
// group-major, then (sequence, KV head), then z within the group -- so the
// items of one (sequence, head) that read nearly the same keys are dealt to
// neighbouring CTAs, run at the same time and share their K/V tiles in L2,
// while the order stays heaviest first.
constexpr int kZGroup = 2;

__device__ __forceinline__ void tc_item_coords(const PrefillParams &p, int i, int &z, int &b, int &kvh) {
    const int per_group = kZGroup * p.Hkv * p.B;
    const int zg = i / per_group, rem = i - zg * per_group;
    const int pair = rem / kZGroup;
    z = zg * kZGroup + (rem - pair * kZGroup);
    b = pair / p.Hkv;
    kvh = pair - b * p.Hkv;
}

// Returns false for items past a sequence's rows or of a sequence whose
// lengths are inconsistent (*bad set for the latter).
__device__ __forceinline__ bool tc_item(const PrefillParams &p, int i, TcItem &it, bool *bad) {
    int z;
    tc_item_coords(p, i, z, it.b, it.kvh);
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
// barrier's phase runs on across items, and the next item's Q rows are
// fetched (cp.async) as soon as the current item's last S product is done.
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
    // s_full p_full o_done q_full o_free
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
            mbar_init(p_full(x), 2 * kWarpsPerTile);
            mbar_init(o_done(x), 1);
            mbar_init(q_full(x), 2 * kWarpsPerTile);
            mbar_init(o_free(x), 2 * kWarpsPerTile);
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
                int z, b, kvh;
                tc_item_coords(p, i, z, b, kvh);
                if (z == 0 && kvh == 0) {
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
        // O_x (+)= P_x . V, P_x from TMEM: the P of keys [64 h, 64 h + 64) sits at
        // columns [64 h, 64 h + 32) of S_x (each softmax half over its own scores)
        const auto issue_pv = [&](int x, int stage, bool acc) {
            const uint32_t vbase = smem_u32(smem + Geo::kV + stage * Geo::kKVBytes);
#pragma unroll
            for (int k = 0; k < kKeys / 16; ++k)
                tc::mma_ts(tmem + Geo::kO + D * x, tmem + kKeys * x + 64 * (k / 4) + 8 * (k % 4),
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
                if (ok && lane == 0) issue_s(x, gk % KS);
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
                if (ok && lane == 0) tc::commit(o_done(x));
                __syncwarp();
            }
            k = kn;
        }
    } else {
        // ---------------- softmax warps.  Tile x has two warpgroups: half hf
        // takes keys [64 hf, 64 hf + 64) of every key tile (P columns
        // [32 hf, 32 hf + 32)) and O columns [hf D / 2, (hf + 1) D / 2) for
        // the rescale and the epilogue; thread t of either half = TMEM lane t
        // = row r_begin + 128 x + t.  Per key tile the halves exchange their
        // row maxima (and at the end of an item their row sums) through
        // shared memory behind the tile's named barrier, which also carries
        // each warp's "wait gave up" vote so that all eight warps of a tile
        // leave the loop at the same step.
        const int tile = warp / (2 * kWarpsPerTile);
        const int hf = (warp / kWarpsPerTile) & 1;
        const int t = threadIdx.x & (kRows - 1);
        const int wq = warp & (2 * kWarpsPerTile - 1);  // warp within the tile: vote slot
        const uint32_t lane_addr = static_cast<uint32_t>((warp % kWarpsPerTile) * 32) << 16;
        const uint32_t t_s = tmem + lane_addr + kKeys * tile;
        const uint32_t t_o = tmem + lane_addr + Geo::kO + D * tile;
        uint8_t *qrow = smem + Geo::kQ + tile * Geo::kQBytes + t * 128;
        float *xch = reinterpret_cast<float *>(smem + Geo::kXch) + tile * Geo::kXchPerTile;
        // xch: max [2 step parities][2 halves][128 rows], sum [2 item parities][2 halves][128
        // rows], votes [2 step parities + 2 item parities][8 warps].  Alternate slots: a
        // slot is written again only after a later barrier that the partner half passes
        // after reading it.
        float *x_max = xch, *x_sum = xch + 4 * kRows;
        volatile int *x_vote = reinterpret_cast<volatile int *>(xch + 8 * kRows);
        const auto tile_bar = [&]() {  // the 256 threads of this tile's two halves
            asm volatile("bar.sync %0, %1;" ::"r"(1 + tile), "r"(2 * kWarpsPerTile * 32) : "memory");
        };
        // every warp of the tile votes in vote slot `slot`; true if all eight are still fine
        const auto tile_vote = [&](bool fine, int slot) {
            if (lane == 0) x_vote[8 * slot + wq] = fine ? 1 : 0;
            tile_bar();
            bool all = true;
#pragma unroll
            for (int w = 0; w < 2 * kWarpsPerTile; ++w) all = all && x_vote[8 * slot + w] != 0;
            return all;
        };
        // this thread's half of its Q row of an item into shared memory
        // (K-major, 128-byte swizzle; rows past the item's rows are zero-filled)
        const auto fetch_q = [&](const TcItem &nx) {
            const int r = nx.r_begin + tile * kRows + t;
            const __nv_bfloat16 *src = p.q;
            uint32_t bytes = 0;
            if (r < nx.rows) {
                src = p.q + (static_cast<size_t>(nx.q0 + r / G) * p.Hq + nx.kvh * G + r % G) * D;
                bytes = 16;
            }
#pragma unroll
            for (int c = hf * (D / 16); c < (hf + 1) * (D / 16); ++c)
                cp_async16(smem_u32(qrow + (c >> 3) * (kRows * 128) + (((c & 7) ^ (t & 7)) << 4)),
                           src + (bytes ? c * 8 : 0), bytes);
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
        const auto publish_q = [&]() {  // the fetched rows, to the tensor core
            asm volatile("cp.async.wait_all;" ::: "memory");
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_full(tile));
        };
        bool ok = true;
        int ns = 0;    // S products seen (s_full / p_full phases; vote parity)
        int n_it = 0;  // items done (o_done phases)
        TcItem it, nx;  // the current and the next item
        int k = tc_next_item(p, 0, it);
        if (k >= 0) {
            fetch_q(it);
            publish_q();
        }
        while (k >= 0 && ok) {
            const int kn = tc_next_item(p, k + 1, nx);
            const int r = it.r_begin + tile * kRows + t;
            const int row_pos = r < it.rows ? it.first_pos + r / G : -1;
            const int my_nk = tile == 0 ? it.nk0 : it.nk1;
            __nv_bfloat16 *out_row =
                p.out + (static_cast<size_t>(it.q0 + r / G) * p.Hq + it.kvh * G + r % G) * D;
            float m_run = -INFINITY, l_run = 0.f;  // l_run: this half's keys
            if (my_nk == 0 && kn >= 0) fetch_q(nx);
            for (int j = 0; j < my_nk; ++j, ++ns) {
                // S_x(j) done; it was issued after PV_x(j - 1), so O_x is free too
                const bool got = mbar_wait(s_full(tile), static_cast<uint32_t>(ns & 1), kWaitLimitNs) &&
                                 !*abort_flag;
                tc::fence_after();
                // this half's 64 scores of the row, 32 at a time (two passes: the
                // row max, then P), causal mask by position
                const int k0 = j * kKeys + 64 * hf;
                const bool masked = __any_sync(0xffffffffu, k0 + 63 > row_pos);
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if (got) {
#pragma unroll 1
                    for (int q = 0; q < 2; ++q) {
                        uint32_t sr[32];
                        tc::ld32(t_s + 64 * hf + 32 * q, sr);
                        tc::wait_ld();
                        if (masked) {
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (k0 + 32 * q + c > row_pos) sr[c] = 0xFF800000u;  // -inf
                        }
#pragma unroll
                        for (int c = 0; c < 32; c += 2)
                            mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
                    }
                }
                x_max[(2 * (ns & 1) + hf) * kRows + t] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                if (!tile_vote(got, ns & 1)) {
                    ok = false;
                    break;
                }
                // the last S product of this item has read Q_x: fetch the next item's rows
                if (j + 1 == my_nk && kn >= 0) fetch_q(nx);
                // row max of the raw scores (scale > 0), both halves
                const float mx = fmaxf(x_max[(2 * (ns & 1)) * kRows + t], x_max[(2 * (ns & 1) + 1) * kRows + t]) *
                                 p.scale_log2;
                // keep the running max unless it grows by more than 2^8 (the same
                // decision in both halves: the same inputs)
                const bool grow = mx > m_run + kRescaleThreshold || (m_run == -INFINITY && mx != -INFINITY);
                const float m_new = grow ? mx : m_run;
                const float nbase = m_new == -INFINITY ? 0.f : -m_new;
                // P of this half's 64 keys, 32 columns (two keys per column), 16 at a time
                const uint64_t scale2 = f2pack(p.scale_log2, p.scale_log2);
                const uint64_t nbase2 = f2pack(nbase, nbase);
                uint64_t sum2[2] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
#pragma unroll 1
                for (int q = 0; q < 2; ++q) {
                    uint32_t sr[32];
                    tc::ld32(t_s + 64 * hf + 32 * q, sr);
                    tc::wait_ld();
                    if (masked) {  // diagonal tiles: -inf scores (2^-inf = 0)
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (k0 + 32 * q + c > row_pos) sr[c] = 0xFF800000u;
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {  // scale and shift two at a time, 2^x on the SFU
                        float a, bb;
                        f2unpack(ffma2(f2pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), scale2, nbase2), a, bb);
                        if ((c >> 1) % 16 < kFmaExpPairs) {
                            exp2_fma2(a, bb);
                        } else {
                            a = ex2_approx(a);
                            bb = ex2_approx(bb);
                        }
                        sum2[(c >> 1) & 1] = fadd2(sum2[(c >> 1) & 1], f2pack(a, bb));
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(a, bb);
                        pk[c / 2] = *reinterpret_cast<uint32_t *>(&h2);
                    }
                    // P over this half's own S columns, already read: keys [64 hf, 64 hf + 64)
                    // at columns [64 hf, 64 hf + 32) -- never over the other half's scores
                    tc::st16(t_s + 64 * hf + 16 * q, pk);
                }
                float s_lo, s_hi, s_lo2, s_hi2;
                f2unpack(sum2[0], s_lo, s_hi);
                f2unpack(sum2[1], s_lo2, s_hi2);
                const float rowsum = (s_lo + s_hi) + (s_lo2 + s_hi2);
                if (j > 0) {
                    const float alpha = (grow && m_run != -INFINITY) ? exp2f(m_run - m_new) : 1.f;
                    if (__any_sync(0xffffffffu, alpha != 1.f)) {  // this half's columns of O
#pragma unroll
                        for (int cc = 0; cc < D / 64; ++cc) {
                            uint32_t o[32];
                            tc::ld32(t_o + hf * (D / 2) + 32 * cc, o);
                            tc::wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                            tc::st32(t_o + hf * (D / 2) + 32 * cc, o);
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
                // This tile's S products of the item are all done, so the tensor
                // core has taken this item's Q phase: the next one may be posted.
                if (j + 1 == my_nk && kn >= 0) publish_q();
            }
            if (!ok) break;
            // O_x of this item complete (a tile without rows gets a bare commit)
            const bool done = mbar_wait(o_done(tile), static_cast<uint32_t>(n_it & 1), kWaitLimitNs) &&
                              !*abort_flag;
            tc::fence_after();
            float *sums = x_sum + 2 * kRows * (n_it & 1);
            sums[hf * kRows + t] = l_run;
            if (!tile_vote(done, 2 + (n_it & 1))) {
                ok = false;
                break;
            }
            const float l_row = sums[t] + sums[kRows + t];
            if (my_nk == 0 && kn >= 0) publish_q();  // after o_done: at most one phase ahead
            ++n_it;
            if (my_nk == 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(o_free(tile));
                it = nx;
                k = kn;
                continue;
            }
            // this half's O columns of the row, normalised, packed to bf16 and
            // stored; then O_x is handed back
            const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
            uint4 *dst = reinterpret_cast<uint4 *>(out_row) + hf * (D / 16);
#pragma unroll 1
            for (int cc = 0; cc < D / 64; ++cc) {
                uint32_t o[32];
                tc::ld32(t_o + hf * (D / 2) + 32 * cc, o);
                tc::wait_ld();
                if (row_pos >= 0) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[8 * i + 2 * e]) * inv,
                                                                      __uint_as_float(o[8 * i + 2 * e + 1]) * inv);
                            w[e] = *reinterpret_cast<uint32_t *>(&h2);
                        }
                        dst[4 * cc + i] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free(tile));
            it = nx;
            k = kn;
        }
        if (!ok && t == 0 && hf == 0) {
            flag(p.err, PKV_DEV_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
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
    const long long zlevels = (rows + kCtaRows - 1) / kCtaRows;
    const long long items = (zlevels + kZGroup - 1) / kZGroup * kZGroup * p.Hkv * p.B;
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
