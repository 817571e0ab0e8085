// Shared-prefix ("cascade") decode attention.
//
// Several sequences whose block tables start with the same physical blocks
// ("vLLM 與 PagedAttention：高吞吐推理的關鍵", section 二, 無法共享: the tables of
// requests with a common prefix point at one set of blocks) need the same
// prefix K/V.  Plain decode streams those shared blocks once per sequence;
// here they are read once per (group, KV head) and the attention of every
// member's query against them is computed as one dense product:
//   rows = (member, query head of this KV head) pairs, 16 per warp tile,
//   S[16 rows x 16 tokens] = Q . K_blk^T  and  O[16 x d] += P . V_blk
// on mma.m16n8k16 (bf16 in, fp32 accumulate) -- with 128 members this is a
// 128-row tile per KV head, a real dense contraction.  (The same chunk runs
// on tcgen05 with TMEM accumulators when selected: prefix_unit_tc below.)
// Each CTA takes a chunk of CB prefix blocks, loads its K and V tiles once
// with TMA, and leaves one partial (m, l, o) per row.  The private suffixes go through the split-K
// kernel starting past the prefix, and the merge below combines prefix and
// suffix partials of each (sequence, query head) by log-sum-exp.  The result
// equals plain decode over the whole sequence.
#include <algorithm>

#include "decode_unit.cuh"
#include "tcgen05.cuh"

namespace pkv {

namespace {

using namespace dev;

constexpr int kPrefixWarps = 4;
constexpr float kLazyRescale = 8.0f;  // log2 units: the running max moves past this growth only

template <int D, int CB>
struct PrefixMmaGeometry {
    static constexpr int kTile = (D / 64) * kBoxBytes;  // one K or V tile of a block
    static constexpr int kSmemBytes = 2 * CB * kTile + 8 + CB * 4 + 1024;
};

// Prefix chunk c (blocks [c*CB, (c+1)*CB) of group g's shared prefix) for KV
// head kvh: all member rows against the chunk's K/V, one partial per row.
template <int D, int CB>
__device__ __forceinline__ void prefix_unit_mma(const CUtensorMap &tmk, const CUtensorMap &tmv,
                                            const PrefixParams &p, int c, int kvh, int g) {
    constexpr int KS = D / 16;                     // k-steps of S = Q K^T over d
    constexpr int NT = D / 8;                      // 8-column tiles of O
    constexpr int kTile = PrefixMmaGeometry<D, CB>::kTile;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tig = lane & 3, gid = lane >> 2;

    const int off = __ldg(p.group_offsets + g);
    const int members = __ldg(p.group_offsets + g + 1) - off;
    if (members <= 0) return;
    const int b0 = __ldg(p.group_seqs + off);
    if (b0 < 0 || b0 >= p.B) {
        if (threadIdx.x == 0) flag(p.err, PKV_DEV_ERR_BAD_LEN);
        return;
    }
    int len0 = __ldg(p.seq_lens + b0);
    len0 = len0 < 0 ? 0 : min(len0, p.W * kBlockTokens);
    const int nb = min(max(__ldg(p.prefix_blocks + b0), 0), len0 / kBlockTokens);  // full blocks
    const int j0 = c * CB, j1 = min(nb, j0 + CB);
    if (j0 >= j1) return;
    const int nt = j1 - j0;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ktiles = smem;                    // [CB][kTile]
    uint8_t *vtiles = smem + CB * kTile;       // [CB][kTile]
    const uint32_t bar = smem_u32(smem + 2 * CB * kTile);
    int *valid = reinterpret_cast<int *>(smem + 2 * CB * kTile + 8);  // [CB]

    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const int32_t *row = p.block_tables + static_cast<size_t>(b0) * p.W;
        uint32_t bytes = 0;
        for (int t = 0; t < nt; ++t) {
            const int32_t phys = __ldg(row + j0 + t);
            valid[t] = phys >= 0 && phys < p.num_blocks ? phys : -1;
            if (valid[t] >= 0) bytes += 2 * kTile;
        }
        mbar_arrive_expect_tx(bar, bytes);
        const uint64_t policy = l2_policy_evict_first();
        for (int t = 0; t < nt; ++t) {
            if (valid[t] < 0) {
                flag(p.err, PKV_DEV_ERR_BAD_BLOCK);
                continue;
            }
            const int y = valid[t] * (p.Hkv * kBlockTokens) + kvh * kBlockTokens;
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh) {
                tma_load_2d(smem_u32(ktiles + t * kTile) + hh * kBoxBytes, &tmk, hh * 64, y, bar, policy);
                tma_load_2d(smem_u32(vtiles + t * kTile) + hh * kBoxBytes, &tmv, hh * 64, y, bar, policy);
            }
        }
    }
    __syncthreads();  // valid[] written
    if (!mbar_wait(bar, 0, kWaitLimitNs)) {
        if (threadIdx.x == 0) flag(p.err, PKV_DEV_ERR_TIMEOUT);
        mbar_wait(bar, 0, kWaitLimitNs);  // let copies in flight land before exiting
        return;
    }

    const int G = p.group;        // query heads per KV head
    const int R = members * G;    // query rows of this group and KV head
    for (int rt = warp; rt * 16 < R; rt += kPrefixWarps) {
        // Q rows (member, head) as mma A fragments: rows gid and gid + 8.
        int rb[2], rh[2];
        const uint32_t *qr[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = rt * 16 + gid + 8 * i;
            rb[i] = -1;
            rh[i] = 0;
            qr[i] = nullptr;
            if (r < R) {
                const int b = __ldg(p.group_seqs + off + r / G);
                if (b >= 0 && b < p.B) {
                    rb[i] = b;
                    rh[i] = kvh * G + r % G;
                    qr[i] = reinterpret_cast<const uint32_t *>(p.q + (static_cast<size_t>(b) * p.Hq + rh[i]) * D);
                }
            }
        }
        uint32_t qa[KS][4];
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            qa[ks][0] = qr[0] ? __ldg(qr[0] + (16 * ks + 2 * tig) / 2) : 0u;
            qa[ks][1] = qr[1] ? __ldg(qr[1] + (16 * ks + 2 * tig) / 2) : 0u;
            qa[ks][2] = qr[0] ? __ldg(qr[0] + (16 * ks + 8 + 2 * tig) / 2) : 0u;
            qa[ks][3] = qr[1] ? __ldg(qr[1] + (16 * ks + 8 + 2 * tig) / 2) : 0u;
        }
        float o[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) o[n][i] = 0.f;
        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

        // Two blocks (32 tokens) per step: S for both, one row-max update,
        // one (rare) rescale, then P.V for each block.  The running max only
        // moves when a row's max grows by more than 2^8, so O is rescaled
        // seldom and P stays <= 2^8; the partial's m is that base.
        for (int t0 = 0; t0 < nt; t0 += 2) {
            const bool v0 = valid[t0] >= 0, v1 = t0 + 1 < nt && valid[t0 + 1] >= 0;
            float s[4][4];  // 8-token column tiles: block t0 tokens 0-7, 8-15, block t0+1 0-7, 8-15
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) s[n][i] = 0.f;
            {
                const int tok = (lane & 7) + (lane >> 4) * 8;
                const int cb = (lane >> 3) & 1;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (!(half ? v1 : v0)) continue;
                    const uint32_t kt = smem_u32(ktiles + (t0 + half) * kTile);
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        uint32_t b00, b01, b10, b11;
                        ldmatrix_x4(kt + tile_off(tok, 2 * ks + cb), b00, b01, b10, b11);
                        mma_bf16_16816(s[2 * half], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b00, b01);
                        mma_bf16_16816(s[2 * half + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b10, b11);
                    }
                }
            }
            // scores in the exp2 domain; a block that is not there scores -inf
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const bool there = n < 2 ? v0 : v1;
#pragma unroll
                for (int i = 0; i < 4; ++i) s[n][i] = there ? s[n][i] * p.scale_log2 : -INFINITY;
            }
            // row gid: s[n][0], s[n][1]; row gid + 8: s[n][2], s[n][3]
            float mx0 = fmaxf(fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1])),
                              fmaxf(fmaxf(s[2][0], s[2][1]), fmaxf(s[3][0], s[3][1])));
            float mx1 = fmaxf(fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3])),
                              fmaxf(fmaxf(s[2][2], s[2][3]), fmaxf(s[3][2], s[3][3])));
#pragma unroll
            for (int m = 1; m < 4; m <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, m));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, m));
            }
            const bool g0 = mx0 > m_run[0] + kLazyRescale || (m_run[0] == -INFINITY && mx0 != -INFINITY);
            const bool g1 = mx1 > m_run[1] + kLazyRescale || (m_run[1] == -INFINITY && mx1 != -INFINITY);
            const float al0 = g0 && m_run[0] != -INFINITY ? ex2_approx(m_run[0] - mx0) : 1.f;
            const float al1 = g1 && m_run[1] != -INFINITY ? ex2_approx(m_run[1] - mx1) : 1.f;
            if (g0) m_run[0] = mx0;
            if (g1) m_run[1] = mx1;
            if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    o[n][0] *= al0;
                    o[n][1] *= al0;
                    o[n][2] *= al1;
                    o[n][3] *= al1;
                }
            }
            const float nb0 = m_run[0] == -INFINITY ? 0.f : m_run[0];
            const float nb1 = m_run[1] == -INFINITY ? 0.f : m_run[1];
            float pr[4][4];
            float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                pr[n][0] = ex2_approx(s[n][0] - nb0);
                pr[n][1] = ex2_approx(s[n][1] - nb0);
                pr[n][2] = ex2_approx(s[n][2] - nb1);
                pr[n][3] = ex2_approx(s[n][3] - nb1);
                sum0 += pr[n][0] + pr[n][1];
                sum1 += pr[n][2] + pr[n][3];
            }
            l_run[0] = l_run[0] * al0 + sum0;
            l_run[1] = l_run[1] * al1 + sum1;
            const int tok = (lane & 7) + ((lane >> 3) & 1) * 8;
            const int cb = lane >> 4;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (!(half ? v1 : v0)) continue;
                const uint32_t vt = smem_u32(vtiles + (t0 + half) * kTile);
                const uint32_t pa0 = pack_bf16x2(pr[2 * half][0], pr[2 * half][1]);
                const uint32_t pa1 = pack_bf16x2(pr[2 * half][2], pr[2 * half][3]);
                const uint32_t pa2 = pack_bf16x2(pr[2 * half + 1][0], pr[2 * half + 1][1]);
                const uint32_t pa3 = pack_bf16x2(pr[2 * half + 1][2], pr[2 * half + 1][3]);
#pragma unroll
                for (int i = 0; i < NT / 2; ++i) {
                    uint32_t w0, w1, w2, w3;
                    ldmatrix_x4_trans(vt + tile_off(tok, 2 * i + cb), w0, w1, w2, w3);
                    mma_bf16_16816(o[2 * i], pa0, pa1, pa2, pa3, w0, w1);
                    mma_bf16_16816(o[2 * i + 1], pa0, pa1, pa2, pa3, w2, w3);
                }
            }
        }
#pragma unroll
        for (int m = 1; m < 4; m <<= 1) {
            l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], m);
            l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], m);
        }
        // partial of (sequence, head) for prefix chunk c
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if (rb[i] < 0) continue;
            const size_t slot = (static_cast<size_t>(rb[i]) * p.Hq + rh[i]) * p.ws_parts + c;
            float *dst = p.ws_o + slot * D;
#pragma unroll
            for (int n = 0; n < NT; ++n)
                *reinterpret_cast<float2 *>(dst + 8 * n + 2 * tig) = make_float2(o[n][2 * i], o[n][2 * i + 1]);
            if (tig == 0) {
                p.ws_ml[2 * slot] = m_run[i];
                p.ws_ml[2 * slot + 1] = l_run[i];
            }
        }
    }
}

template <int D, int CB>
struct PrefixTcGeometry {
    static constexpr int kKeys = CB * kBlockTokens;     // keys of one chunk: MMA N of S, K of P.V
    static constexpr int kKV = (D / 64) * kKeys * 128;  // one K or V chunk [d half][key][128 B]
    static constexpr int kQ = (D / 64) * 128 * 128;     // one 128-row Q tile [d half][row][128 B]
    static constexpr int kMeta = 64;                    // 3 mbarriers, TMEM base, keep bits x 2
    static constexpr int kSmemBytes = 2 * kKV + kQ + kMeta + 1024;
    static constexpr int kTmemCols = 256;               // S (P over its first half) | O
    static_assert(kKeys % 64 == 0 && kKeys <= 128 && CB <= 32, "chunk layout");
    static_assert(kKeys + D <= kTmemCols, "tensor memory columns");
};

// Prefix range c of group g's shared prefix -- chunks [c * RC, (c + 1) * RC)
// of CB blocks each, RC = p.range_blocks / CB -- for KV head kvh, on the tcgen05
// tensor cores.  The rows, (member, query head) pairs, go in tiles of 128,
// one row per thread (= TMEM lane); for each row tile the range's chunks run
// one after another with an online softmax:
//   S[128 x 16 CB] = Q K^T        tcgen05.mma, Q tile and K chunk in shared memory
//   m = running row max (moved only when it grows by more than 2^8),
//   P = 2^(S * scale - m) as bf16 into TMEM over S, l += sum P,
//   O in TMEM rescaled by 2^(m_old - m) when the max moves
//   O[128 x d] (+)= P V           tcgen05.mma, P from TMEM, V chunk in shared memory
// (chunks of 4 blocks keep the CTA's shared memory -- K chunk, V chunk, Q
// tile -- near a suffix CTA's, so that a prefix CTA displaces one of them)
// and leaves one partial (m, l, O) per row for the range.  The next chunk's K
// is loaded as soon as S has read this one, its V as soon as P.V has, so the
// loads overlap the softmax.  Keys of blocks past the prefix or with a bad
// table entry load as zeros (a row past the tensor) and are masked.  Every
// wait is bounded; on a timeout the CTA flags it, waits (bounded) for its
// copies and MMAs, and frees its TMEM.
template <int D, int CB>
__device__ __forceinline__ void prefix_range_tc(const CUtensorMap &tmk, const CUtensorMap &tmv,
                                                const PrefixParams &p, int c, int kvh, int g) {
    using Geo = PrefixTcGeometry<D, CB>;
    constexpr int kKeys = Geo::kKeys;
    constexpr int kColS = 0, kColO = kKeys;  // TMEM columns
    constexpr uint32_t kIdS = tc::idesc_bf16(128, kKeys, 0);
    constexpr uint32_t kIdO = tc::idesc_bf16(128, D, 1);
    const int t = threadIdx.x, warp = t >> 5;

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
    const int rc = p.range_blocks / CB;  // chunks per range
    const int c0 = c * rc, c1 = min((nb + CB - 1) / CB, c0 + rc);
    if (c0 >= c1) return;
    const int nc = c1 - c0;          // chunks of the range
    const int G = p.group;           // query heads per KV head
    const int R = members * G;       // rows of this group and KV head
    const int steps = ((R + 127) / 128) * nc;  // (row tile, chunk), chunk fastest

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t k_smem = smem_u32(smem), v_smem = smem_u32(smem + Geo::kKV);
    uint8_t *q_tile = smem + 2 * Geo::kKV;
    uint8_t *meta = q_tile + Geo::kQ;
    const uint32_t k_bar = smem_u32(meta);  // a K chunk landed
    const uint32_t v_bar = k_bar + 8;       // a V chunk landed
    const uint32_t m_bar = k_bar + 16;      // the MMAs issued so far are done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(meta + 24);
    volatile uint32_t *keep_bits = reinterpret_cast<volatile uint32_t *>(meta + 32);  // [2], by step parity

    const int32_t *trow = p.block_tables + static_cast<size_t>(b0) * p.W;
    // Thread 0: the TMA loads of chunk `ch` into one buffer; bit i of the
    // return value: block i of the chunk is there.
    const auto load_chunk = [&](int ch, uint32_t dst, uint32_t bar, const CUtensorMap *tm) {
        const int j0 = ch * CB;
        uint32_t keep = 0;
        mbar_arrive_expect_tx(bar, Geo::kKV);
        const uint64_t policy = l2_policy_evict_first();
        const long long y_none = p.num_blocks * p.Hkv * kBlockTokens;  // past the tensor: zeros
#pragma unroll 1
        for (int i = 0; i < CB; ++i) {
            long long y = y_none;
            if (j0 + i < nb) {
                const int32_t phys = __ldg(trow + j0 + i);
                if (phys >= 0 && phys < p.num_blocks) {
                    y = (static_cast<long long>(phys) * p.Hkv + kvh) * kBlockTokens;
                    keep |= 1u << i;
                } else if (tm == &tmk) {
                    flag(p.err, PKV_DEV_ERR_BAD_BLOCK);
                }
            }
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh)
                tma_load_2d(dst + hh * (kKeys * 128) + i * (kBlockTokens * 128), tm, hh * 64,
                            static_cast<int>(y), bar, policy);
        }
        return keep;
    };
    const auto chunk_of = [&](int st) { return c0 + st % nc; };

    if (t == 0) {
        mbar_init(k_bar, 1);
        mbar_init(v_bar, 1);
        mbar_init(m_bar, 1);
        fence_mbar_init();
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        keep_bits[0] = load_chunk(c0, k_smem, k_bar, &tmk);
        load_chunk(c0, v_smem, v_bar, &tmv);
    }
    if (warp == 1) tc::alloc<Geo::kTmemCols>(smem_u32(tmem_slot));  // beside thread 0's TMA issue
    tc::fence_before();
    __syncthreads();  // barriers, keep bits and the TMEM base
    tc::fence_after();
    // Only now may the suffix grid launch: every prefix CTA holds its TMEM
    // before any suffix or merge CTA exists.  (A co-resident CTA that keeps
    // its right to allocate can hold up tcgen05.alloc, and suffix CTAs wait
    // for this grid before they exit: allocating after them could wait for
    // ever.)
    pdl_launch_dependents();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);  // this thread's lane

    bool ok = true;
    bool mma_pending = false;  // an MMA batch committed to m_bar and not yet seen done
    uint32_t m_phase = 0;
    int k_issued = 1, k_done = 0, v_issued = 1, v_done = 0;  // chunk loads per buffer (thread 0's view)
    int b = -1, h = 0;  // this thread's row of the current row tile
    float m_run = -INFINITY, l_run = 0.f;
    for (int st = 0; st < steps && ok; ++st) {
        const int ci = st % nc;  // chunk index within the range
        const int ch = c0 + ci;
        const bool new_k = st == 0 || ch != chunk_of(st - 1);  // a load was issued for this step
        const bool new_v = new_k;
        if (ci == 0) {
            // A new row tile: this thread's Q row into the swizzled Q tile (the
            // S product that read the previous tile is done), zeros for rows
            // without a sequence.
            const int r = (st / nc) * 128 + t;
            b = -1;
            h = 0;
            if (r < R) {
                const int bb = __ldg(p.group_seqs + off + r / G);
                if (bb >= 0 && bb < p.B) {
                    b = bb;
                    h = kvh * G + r % G;
                }
            }
            const uint4 *src = reinterpret_cast<const uint4 *>(
                p.q + (static_cast<size_t>(b < 0 ? 0 : b) * p.Hq + h) * D);
            uint8_t *qrow = q_tile + t * 128;
#pragma unroll
            for (int cc = 0; cc < D / 8; ++cc) {
                const uint4 v = b >= 0 ? __ldg(src + cc) : make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4 *>(qrow + (cc >> 3) * (128 * 128) + (((cc & 7) ^ (t & 7)) << 4)) = v;
            }
            fence_proxy_async_smem();  // the generic-proxy stores, before the MMA's reads
            m_run = -INFINITY;
            l_run = 0.f;
        }
        const bool k_ok = !new_k || mbar_wait(k_bar, static_cast<uint32_t>(k_done & 1), kWaitLimitNs);
        if (new_k && k_ok) ++k_done;
        if (__syncthreads_or(!k_ok)) {
            ok = false;
            break;
        }
        tc::fence_after();
        if (t == 0) {  // S = Q K^T
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const int hh = k >> 2, kk = k & 3;
                tc::mma_ss(tmem + kColS,
                           tc::smem_desc(smem_u32(q_tile) + hh * (128 * 128) + kk * 32, 16, 1024),
                           tc::smem_desc(k_smem + hh * (kKeys * 128) + kk * 32, 16, 1024), kIdS, k > 0);
            }
            tc::commit(m_bar);
        }
        mma_pending = true;
        if (__syncthreads_or(!mbar_wait(m_bar, m_phase, kWaitLimitNs))) {
            ok = false;
            break;
        }
        mma_pending = false;
        m_phase ^= 1;
        tc::fence_after();
        // S has read this K chunk: the next step's K may come in now
        if (st + 1 < steps && chunk_of(st + 1) != ch) {
            if (t == 0) keep_bits[(st + 1) & 1] = load_chunk(chunk_of(st + 1), k_smem, k_bar, &tmk);
            ++k_issued;
        } else if (t == 0 && st + 1 < steps) {
            keep_bits[(st + 1) & 1] = keep_bits[st & 1];
        }
        const uint32_t keep = keep_bits[st & 1];

        // softmax of the row, two passes over S (64 columns at a time): max, then P
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
        for (int hf = 0; hf < kKeys / 64; ++hf) {
            uint32_t sv[64];
            tc::ld32(lane_base + kColS + 64 * hf, sv);
            tc::ld32(lane_base + kColS + 64 * hf + 32, sv + 32);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 64; ++i)
                if (keep >> (4 * hf + i / kBlockTokens) & 1u)
                    mx4[i / kBlockTokens] = fmaxf(mx4[i / kBlockTokens], __uint_as_float(sv[i]) * p.scale_log2);
        }
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        const bool grow = mx > m_run + kLazyRescale || (m_run == -INFINITY && mx != -INFINITY);
        const float m_new = grow ? mx : m_run;
        const float nbase = m_new == -INFINITY ? 0.f : m_new;
        float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int hf = 0; hf < kKeys / 64; ++hf) {
            uint32_t sv[64];
            tc::ld32(lane_base + kColS + 64 * hf, sv);
            tc::ld32(lane_base + kColS + 64 * hf + 32, sv + 32);
            tc::wait_ld();
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
                const bool there = keep >> (4 * hf + i / kBlockTokens) & 1u;  // i, i + 1: one block
                const float p0 = there ? ex2_approx(fmaf(__uint_as_float(sv[i]), p.scale_log2, -nbase)) : 0.f;
                const float p1 = there ? ex2_approx(fmaf(__uint_as_float(sv[i + 1]), p.scale_log2, -nbase)) : 0.f;
                l4[i / kBlockTokens] += p0 + p1;
                pk[i / 2] = pack_bf16x2(p0, p1);
            }
            tc::st32(lane_base + kColS + 32 * hf, pk);  // P columns over S columns already read
        }
        const float alpha = (ci > 0 && grow && m_run != -INFINITY) ? exp2f(m_run - m_new) : 1.f;
        if (__any_sync(0xffffffffu, alpha != 1.f)) {  // O of the earlier chunks, to the new max
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tc::ld32(lane_base + kColO + 32 * cc, o);
                tc::wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                tc::st32(lane_base + kColO + 32 * cc, o);
            }
        }
        l_run = l_run * alpha + ((l4[0] + l4[1]) + (l4[2] + l4[3]));
        m_run = m_new;
        tc::wait_st();
        tc::fence_before();
        const bool v_ok = !new_v || mbar_wait(v_bar, static_cast<uint32_t>(v_done & 1), kWaitLimitNs);
        if (new_v && v_ok) ++v_done;
        if (__syncthreads_or(!v_ok)) {
            ok = false;
            break;
        }
        tc::fence_after();
        if (t == 0) {  // O (+)= P V (V MN-major: d contiguous)
#pragma unroll
            for (int k = 0; k < kKeys / 16; ++k)
                tc::mma_ts(tmem + kColO, tmem + kColS + 8 * k,
                           tc::smem_desc(v_smem + k * (16 * 128), kKeys * 128, 1024), kIdO, ci > 0 || k > 0);
            tc::commit(m_bar);
        }
        mma_pending = true;
        if (__syncthreads_or(!mbar_wait(m_bar, m_phase, kWaitLimitNs))) {
            ok = false;
            break;
        }
        mma_pending = false;
        m_phase ^= 1;
        tc::fence_after();
        // P.V has read this V chunk: the next step's V may come in now
        if (st + 1 < steps && chunk_of(st + 1) != ch) {
            if (t == 0) load_chunk(chunk_of(st + 1), v_smem, v_bar, &tmv);
            ++v_issued;
        }

        if (ci == nc - 1 && b >= 0) {
            // the row's partial for range c: (m, l) and O from TMEM
            const size_t slot = (static_cast<size_t>(b) * p.Hq + h) * p.ws_parts + c;
            p.ws_ml[2 * slot] = m_run;
            p.ws_ml[2 * slot + 1] = l_run;
            float4 *dst = reinterpret_cast<float4 *>(p.ws_o + slot * D);
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tc::ld32(lane_base + kColO + 32 * cc, o);
                tc::wait_ld();
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[8 * cc + i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                                  __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
            }
        }
        tc::fence_before();  // the O reads above, before the next tile's P.V overwrites O
    }
    if (!ok && t == 0) {
        flag(p.err, PKV_DEV_ERR_TIMEOUT);
        if (mma_pending) mbar_wait(m_bar, m_phase, kWaitLimitNs);  // the batch still running
    }
    if (t == 0) {  // a load issued and not waited for (only after a wait gave up): let it land
        if (k_issued > k_done) mbar_wait(k_bar, static_cast<uint32_t>(k_done & 1), kWaitLimitNs);
        if (v_issued > v_done) mbar_wait(v_bar, static_cast<uint32_t>(v_done & 1), kWaitLimitNs);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 1) tc::dealloc<Geo::kTmemCols>(tmem);
}

// Merge of one (sequence, query head): prefix slots [0, ceil(pb / range_blocks)) and
// the suffix split-K partitions that hold tokens past the prefix (counted
// from the prefix end), in slot order, by log-sum-exp.  As in the split-K
// merge: all (m, l) read at once, weights computed once, output loads batched.
template <int D, int CB>
__global__ void __launch_bounds__(D) cascade_merge_kernel(const PrefixParams p) {
    constexpr int kMaxSlots = 256;
    __shared__ float s_w[kMaxSlots];
    __shared__ float s_red[D / 32][2];
    const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
    pdl_wait_primary();  // the cascade grid's partials
    int len = __ldg(p.seq_lens + b);
    len = len < 0 ? 0 : min(len, p.W * kBlockTokens);
    const int nblk = (len + kBlockTokens - 1) / kBlockTokens;
    const int pb = min(max(__ldg(p.prefix_blocks + b), 0), len / kBlockTokens);
    const int nchunks = (pb + p.range_blocks - 1) / p.range_blocks;  // prefix slots
    // suffix partitions with tokens, at most those the launch computed (a
    // longer suffix was flagged by the cascade kernel)
    const int ntot = nchunks + min((nblk - pb + p.part_blocks - 1) / p.part_blocks,
                                   p.ws_parts - p.prefix_parts);
    const auto slot = [&](int q) { return q < nchunks ? q : p.prefix_parts + (q - nchunks); };
    const size_t row = static_cast<size_t>(b) * p.Hq + h;
    const float *ml = p.ws_ml + 2 * row * p.ws_parts;
    const float *o = p.ws_o + row * p.ws_parts * D;
    float mx = -INFINITY;
    for (int q = e; q < ntot; q += D) mx = fmaxf(mx, ml[2 * slot(q)]);
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    if ((e & 31) == 0) s_red[e >> 5][0] = mx;
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) M = fmaxf(M, s_red[w][0]);
    float L = 0.f, O = 0.f;
    for (int base = 0; base < ntot; base += kMaxSlots) {
        const int n = min(kMaxSlots, ntot - base);
        __syncthreads();  // s_w and s_red reuse
        float lsum = 0.f;
        for (int q = e; q < n; q += D) {
            const float2 v = *reinterpret_cast<const float2 *>(ml + 2 * slot(base + q));
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
        int q = 0;
        for (; q + 8 <= n; q += 8) {
            float x[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = o[static_cast<size_t>(slot(base + q + i)) * D + e];
#pragma unroll
            for (int i = 0; i < 8; ++i) O = fmaf(x[i], s_w[q + i], O);
        }
        for (; q < n; ++q) O = fmaf(o[static_cast<size_t>(slot(base + q)) * D + e], s_w[q], O);
    }
    p.out[row * D + e] = __float2bfloat16(L > 0.f ? O / L : 0.f);
}

// The prefix grid: CTA k is prefix range k % prefix_parts of KV head
// (k / prefix_parts) % Hkv of group k / (prefix_parts * Hkv).  It lets the
// suffix grid, launched after it as a programmatic dependent, start early:
// the two run side by side, the short tensor-core prefix work beside the
// bandwidth-bound suffix stream.  TC: ranges on tcgen05 (else one chunk per
// CTA on mma.sync); a tcgen05 CTA lets the suffix grid launch only once it
// holds its tensor memory (in prefix_range_tc), a CTA without prefix work by
// exiting.
template <int D, bool TC>
__global__ void __launch_bounds__(kPrefixWarps * 32)
    cascade_prefix_kernel(const __grid_constant__ CUtensorMap tmk,
                          const __grid_constant__ CUtensorMap tmv, const PrefixParams pp) {
    if constexpr (!TC) pdl_launch_dependents();
    int id = blockIdx.x;
    const int c = id % pp.prefix_parts;
    id /= pp.prefix_parts;
    if constexpr (TC)
        prefix_range_tc<D, kPrefixTcChunkBlocks>(tmk, tmv, pp, c, id % pp.Hkv, id / pp.Hkv);
    else
        prefix_unit_mma<D, kPrefixChunkBlocks>(tmk, tmv, pp, c, id % pp.Hkv, id / pp.Hkv);
}

// The suffix grid: split-K units from each sequence's prefix end (partition
// fastest, then head segment, then sequence).  WIDE: each CTA covers
// kPrefixWarps head segments of one sequence, a warp each (suffixes are
// short: one warp per segment keeps every ring busy for the whole suffix
// instead of a quarter of it).  Before it exits, each CTA waits for the
// prefix grid, so that this grid's completion -- which the merge waits for --
// also covers the prefix partials.
template <int D, bool MMA, bool WIDE>
__global__ void __launch_bounds__(kPrefixWarps * 32)
    cascade_suffix_kernel(const __grid_constant__ CUtensorMap tmk,
                          const __grid_constant__ CUtensorMap tmv, const DecodeParams dp) {
    // These CTAs use no tensor memory: they give up the right to allocate at
    // once, so that they can never hold up a tcgen05.alloc on their SM.
    if (threadIdx.x < 32) tc::relinquish();
    int id = blockIdx.x;
    const int ny = (MMA ? dp.Hkv * dp.chunks : dp.Hq) / (WIDE ? kPrefixWarps : 1);
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
    decode_unit<D, kPrefixWarps, 2, MMA, kModeSplit, WIDE>(tmk, tmv, dp, part, id % ny, b);
    pdl_wait_primary();
}

template <int D, bool MMA, bool TC, bool WIDE>
cudaError_t launch_cascade_d(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefixParams &pp,
                             const DecodeParams &dp, int num_groups, cudaStream_t stream) {
    const long long n_pre = static_cast<long long>(pp.prefix_parts) * pp.Hkv * num_groups;
    const long long ny = (MMA ? dp.Hkv * dp.chunks : dp.Hq) / (WIDE ? kPrefixWarps : 1);
    const long long n_suf = static_cast<long long>(dp.num_parts) * ny * dp.B;
    if (n_pre >= (1ll << 31) || n_suf >= (1ll << 31)) return cudaErrorInvalidValue;
    cudaError_t e;
    if (n_pre > 0) {
        constexpr int kPre = TC ? PrefixTcGeometry<D, kPrefixTcChunkBlocks>::kSmemBytes
                                : PrefixMmaGeometry<D, kPrefixChunkBlocks>::kSmemBytes;
        auto pre = cascade_prefix_kernel<D, TC>;
        if ((e = cudaFuncSetAttribute(pre, cudaFuncAttributeMaxDynamicSharedMemorySize, kPre)) != cudaSuccess)
            return e;
        pre<<<static_cast<unsigned>(n_pre), kPrefixWarps * 32, kPre, stream>>>(tmk, tmv, pp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    constexpr int kSuf = Geometry<D, kPrefixWarps, 2>::kSmemBytes;
    auto suf = cascade_suffix_kernel<D, MMA, WIDE>;
    if ((e = cudaFuncSetAttribute(suf, cudaFuncAttributeMaxDynamicSharedMemorySize, kSuf)) != cudaSuccess)
        return e;
    if (n_suf > 0) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(static_cast<unsigned>(n_suf));
        cfg.blockDim = dim3(kPrefixWarps * 32);
        cfg.dynamicSmemBytes = kSuf;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = n_pre > 0 ? 1 : 0;  // beside the prefix grid
        if ((e = cudaLaunchKernelEx(&cfg, suf, tmk, tmv, dp)) != cudaSuccess) return e;
    }
    return launch_dependent(cascade_merge_kernel<D, kPrefixChunkBlocks>,
                            dim3(static_cast<unsigned>(pp.Hq), static_cast<unsigned>(pp.B)), dim3(D),
                            stream, pp);
}

template <int D, bool TC, bool WIDE>
cudaError_t launch_cascade_w(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefixParams &pp,
                             const DecodeParams &dp, int num_groups, cudaStream_t stream) {
    return dp.group > 1 ? launch_cascade_d<D, true, TC, WIDE>(tmk, tmv, pp, dp, num_groups, stream)
                        : launch_cascade_d<D, false, TC, WIDE>(tmk, tmv, pp, dp, num_groups, stream);
}

template <int D>
cudaError_t launch_cascade_h(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefixParams &pp,
                             const DecodeParams &dp, int num_groups, bool prefix_tc, bool wide,
                             cudaStream_t stream) {
    if (prefix_tc)
        return wide ? launch_cascade_w<D, true, true>(tmk, tmv, pp, dp, num_groups, stream)
                    : launch_cascade_w<D, true, false>(tmk, tmv, pp, dp, num_groups, stream);
    return wide ? launch_cascade_w<D, false, true>(tmk, tmv, pp, dp, num_groups, stream)
                : launch_cascade_w<D, false, false>(tmk, tmv, pp, dp, num_groups, stream);
}

}  // namespace

bool cascade_wide_fits(const DecodeParams &dp) {
    const int segments = dp.group > 1 ? dp.Hkv * dp.chunks : dp.Hq;
    return segments % kPrefixWarps == 0 && dp.chunks == 1;
}

cudaError_t launch_cascade(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefixParams &pp,
                           const DecodeParams &dp, int head_dim, int num_groups, bool prefix_tc,
                           bool wide, cudaStream_t stream) {
    if (wide && !cascade_wide_fits(dp)) return cudaErrorInvalidValue;
    if (head_dim == 128) return launch_cascade_h<128>(tmk, tmv, pp, dp, num_groups, prefix_tc, wide, stream);
    if (head_dim == 64) return launch_cascade_h<64>(tmk, tmv, pp, dp, num_groups, prefix_tc, wide, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pkv
