// Paged prefill attention: causal attention of a sequence's new (prompt)
// tokens over its paged K/V.
//
// "vLLM 與 PagedAttention：高吞吐推理的關鍵", section 三 step 二 (預填充): the
// input tokens' K/V are written into blocks, a new block taken as each one
// fills, and the table updated -- pkv_paged_kv_write with the allocator's
// slots does that part.  Their attention is then over the paged cache: query
// token at position p attends to positions [0, p] of its sequence, which may
// begin with blocks cached before (a shared prefix, or earlier chunks).
//
// Dense work, on tensor cores: rows = (query token, query head of the KV
// head) pairs, 16 per consumer warp and 64 per CTA; for every 16-token block
// S[16 x 16] = Q K^T and O[16 x d] += P V on mma.m16n8k16 (bf16 in, fp32
// accumulate), online softmax per row in the exp2 domain.  One producer warp
// streams the (block, KV head) K/V tiles the CTA's rows can see through a
// shared 4-stage TMA ring (full / empty mbarriers, bounded waits); the four
// consumer warps share every tile.  Key positions past a row's own position
// (causal) or past the sequence end get score -inf, and V rows past the end
// are zeroed before the product so that whatever the tail slots hold never
// reaches the output.
#include "decode_common.cuh"

namespace pkv {

namespace {

using namespace dev;

constexpr int kConsumers = 4;               // consumer warps, 16 rows each
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kRing = 4;                    // TMA stages

template <int D>
struct PrefillGeometry {
    static constexpr int kTile = (D / 64) * kBoxBytes;
    static constexpr int kStage = 2 * kTile;
    static constexpr int kSmemBytes = kRing * kStage + 2 * kRing * 8 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv, const PrefillParams p) {
    using Geo = PrefillGeometry<D>;
    constexpr int KS = D / 16, NT = D / 8;
    const int b = blockIdx.z, kvh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tig = lane & 3, gid = lane >> 2;
    const int G = p.group;

    const int q0 = __ldg(p.query_start + b), q1 = __ldg(p.query_start + b + 1);
    int ctx = __ldg(p.seq_lens + b);
    const int nq = q1 - q0;
    if (nq <= 0 || ctx < nq || ctx > p.W * kBlockTokens) {
        if (nq > 0 && blockIdx.x == 0 && kvh == 0 && threadIdx.x == 0) flag(p.err, PKV_DEV_ERR_BAD_LEN);
        return;
    }
    const int rows = nq * G;
    const int ntiles_q = (rows + 16 * kConsumers - 1) / (16 * kConsumers);
    if (static_cast<int>(blockIdx.x) >= ntiles_q) return;
    const int qt = ntiles_q - 1 - static_cast<int>(blockIdx.x);  // heaviest tiles first
    const int r_begin = qt * 16 * kConsumers;
    const int first_pos = ctx - nq;  // position of query token 0
    // keys this CTA can see: up to the position of its last row
    const int last_row = min(rows, r_begin + 16 * kConsumers) - 1;
    const int kv_end = first_pos + last_row / G + 1;
    const int nblk = (kv_end + kBlockTokens - 1) / kBlockTokens;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t full = smem_u32(smem + kRing * Geo::kStage);
    const uint32_t empty = full + kRing * 8;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kRing; ++s) {
            mbar_init(full + 8 * s, 1);
            mbar_init(empty + 8 * s, kConsumers);
        }
        fence_mbar_init();
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    __syncthreads();
    const int32_t *trow = p.block_tables + static_cast<size_t>(b) * p.W;

    if (warp == kConsumers) {  // ---------------- producer warp
        if (lane == 0) {
            const uint64_t policy = l2_policy_evict_normal();  // tiles are re-read by other CTAs
            for (int j = 0; j < nblk; ++j) {
                const int s = j % kRing;
                if (j >= kRing &&
                    !mbar_wait(empty + 8 * s, static_cast<uint32_t>(((j / kRing) - 1) & 1), kWaitLimitNs)) {
                    flag(p.err, PKV_DEV_ERR_TIMEOUT);
                    break;
                }
                const int32_t phys = __ldg(trow + j);
                if (phys >= 0 && phys < p.num_blocks) {
                    const uint32_t dst = smem_u32(smem + s * Geo::kStage);
                    const int y = phys * (p.Hkv * kBlockTokens) + kvh * kBlockTokens;
                    mbar_arrive_expect_tx(full + 8 * s, Geo::kStage);
#pragma unroll
                    for (int hh = 0; hh < D / 64; ++hh) {
                        tma_load_2d(dst + hh * kBoxBytes, &tmk, hh * 64, y, full + 8 * s, policy);
                        tma_load_2d(dst + Geo::kTile + hh * kBoxBytes, &tmv, hh * 64, y, full + 8 * s, policy);
                    }
                } else {
                    flag(p.err, PKV_DEV_ERR_BAD_BLOCK);
                    mbar_arrive(full + 8 * s);
                }
            }
        }
        return;
    }

    // ---------------- consumer warps: rows r_begin + 16 * warp + [0, 16)
    const int rw = r_begin + 16 * warp;
    int rpos[2];
    const uint32_t *qr[2];
    size_t orow[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = rw + gid + 8 * i;
        rpos[i] = -1;
        qr[i] = nullptr;
        orow[i] = 0;
        if (r < rows) {
            const int t = r / G, h = kvh * G + r % G;
            rpos[i] = first_pos + t;
            orow[i] = (static_cast<size_t>(q0 + t) * p.Hq + h) * D;
            qr[i] = reinterpret_cast<const uint32_t *>(p.q + orow[i]);
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
    // the last key this warp's rows can see
    const int warp_last = min(rows, rw + 16) - 1;
    const int warp_kv_end = rw < rows ? first_pos + warp_last / G + 1 : 0;

    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[n][i] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

    int j = 0;
    for (; j < nblk; ++j) {
        const int s = j % kRing;
        if (!mbar_wait(full + 8 * s, static_cast<uint32_t>((j / kRing) & 1), kWaitLimitNs)) {
            if (lane == 0) flag(p.err, PKV_DEV_ERR_TIMEOUT);
            break;
        }
        const int32_t phys = __ldg(trow + j);
        const int k0 = j * kBlockTokens;
        if (phys >= 0 && phys < p.num_blocks && k0 < warp_kv_end) {
            const uint32_t kt = smem_u32(smem + s * Geo::kStage), vt = kt + Geo::kTile;
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
            {
                const int tok = (lane & 7) + (lane >> 4) * 8;
                const int cb = (lane >> 3) & 1;
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    uint32_t b00, b01, b10, b11;
                    ldmatrix_x4(kt + tile_off(tok, 2 * ks + cb), b00, b01, b10, b11);
                    mma_bf16_16816(s0, qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b00, b01);
                    mma_bf16_16816(s1, qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b10, b11);
                }
            }
            // s0[0..1]: row gid, keys k0 + 2tig + {0,1}; s1: keys + 8; [2..3]: row gid + 8
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = i >> 1;
                const int key0 = k0 + 2 * tig + (i & 1), key1 = key0 + 8;
                s0[i] = (key0 <= rpos[row] && key0 < ctx) ? s0[i] * p.scale_log2 : -INFINITY;
                s1[i] = (key1 <= rpos[row] && key1 < ctx) ? s1[i] * p.scale_log2 : -INFINITY;
            }
            float mx0 = fmaxf(fmaxf(s0[0], s0[1]), fmaxf(s1[0], s1[1]));
            float mx1 = fmaxf(fmaxf(s0[2], s0[3]), fmaxf(s1[2], s1[3]));
#pragma unroll
            for (int m = 1; m < 4; m <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, m));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, m));
            }
            // A row with no visible key in this block (or a padding row) keeps
            // its state: its probabilities are 0 and its scale factor 1.
            const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
            const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m_run[0] - mn0);
            const float al1 = mn1 == -INFINITY ? 1.f : exp2f(m_run[1] - mn1);
            const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
            m_run[0] = mn0;
            m_run[1] = mn1;
            float pr0[4], pr1[4];
            pr0[0] = exp2f(s0[0] - base0);
            pr0[1] = exp2f(s0[1] - base0);
            pr1[0] = exp2f(s1[0] - base0);
            pr1[1] = exp2f(s1[1] - base0);
            pr0[2] = exp2f(s0[2] - base1);
            pr0[3] = exp2f(s0[3] - base1);
            pr1[2] = exp2f(s1[2] - base1);
            pr1[3] = exp2f(s1[3] - base1);
            l_run[0] = l_run[0] * al0 + pr0[0] + pr0[1] + pr1[0] + pr1[1];
            l_run[1] = l_run[1] * al1 + pr0[2] + pr0[3] + pr1[2] + pr1[3];
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                o[n][0] *= al0;
                o[n][1] *= al0;
                o[n][2] *= al1;
                o[n][3] *= al1;
            }
            const uint32_t pa0 = pack_bf16x2(pr0[0], pr0[1]), pa1 = pack_bf16x2(pr0[2], pr0[3]);
            const uint32_t pa2 = pack_bf16x2(pr1[0], pr1[1]), pa3 = pack_bf16x2(pr1[2], pr1[3]);
            // V rows at or past the sequence end: zero (P is 0 there, but 0 * NaN is not)
            const int nvalid = ctx - k0;
            uint32_t keep_lo = 0xFFFFFFFFu, keep_hi = 0xFFFFFFFFu;
            if (nvalid < 16) {
                const int t = 2 * tig;
                keep_lo = (t < nvalid ? 0x0000FFFFu : 0u) | (t + 1 < nvalid ? 0xFFFF0000u : 0u);
                keep_hi = (t + 8 < nvalid ? 0x0000FFFFu : 0u) | (t + 9 < nvalid ? 0xFFFF0000u : 0u);
            }
            const int tok = (lane & 7) + ((lane >> 3) & 1) * 8;
            const int cb = lane >> 4;
#pragma unroll
            for (int i = 0; i < NT / 2; ++i) {
                uint32_t v0, v1, v2, v3;
                ldmatrix_x4_trans(vt + tile_off(tok, 2 * i + cb), v0, v1, v2, v3);
                mma_bf16_16816(o[2 * i], pa0, pa1, pa2, pa3, v0 & keep_lo, v1 & keep_hi);
                mma_bf16_16816(o[2 * i + 1], pa0, pa1, pa2, pa3, v2 & keep_lo, v3 & keep_hi);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + 8 * s);
    }
#pragma unroll
    for (int m = 1; m < 4; m <<= 1) {
        l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], m);
        l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], m);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        if (rpos[i] < 0) continue;
        const float inv = l_run[i] > 0.f ? 1.f / l_run[i] : 0.f;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            __nv_bfloat162 v = __floats2bfloat162_rn(o[n][2 * i] * inv, o[n][2 * i + 1] * inv);
            *reinterpret_cast<__nv_bfloat162 *>(p.out + orow[i] + 8 * n + 2 * tig) = v;
        }
    }
}

template <int D>
cudaError_t launch_prefill_d(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefillParams &p,
                             int max_query_len, cudaStream_t stream) {
    constexpr int kSmem = PrefillGeometry<D>::kSmemBytes;
    auto kern = paged_prefill_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    const long long rows = static_cast<long long>(max_query_len) * p.group;
    const long long tiles = (rows + 16 * kConsumers - 1) / (16 * kConsumers);
    if (tiles == 0) return cudaSuccess;
    if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(p.Hkv),
                    static_cast<unsigned>(p.B));
    kern<<<grid, kThreads, kSmem, stream>>>(tmk, tmv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefillParams &p,
                           int head_dim, int max_query_len, cudaStream_t stream) {
    if (head_dim == 128) return launch_prefill_d<128>(tmk, tmv, p, max_query_len, stream);
    if (head_dim == 64) return launch_prefill_d<64>(tmk, tmv, p, max_query_len, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pkv
