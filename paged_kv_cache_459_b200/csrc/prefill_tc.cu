// Paged prefill attention on the 5th-generation tensor cores (tcgen05, TMEM).
//
// Same result as paged_prefill_kernel (prefill.cu): causal attention of each
// sequence's new tokens over its paged K/V ("vLLM 與 PagedAttention：高吞吐推理
// 的關鍵", section 三 step 二).  A CTA owns 128 query rows -- (token, query
// head of one KV head) pairs -- and walks the keys its rows can see in tiles
// of 64 (four 16-token blocks):
//   S[128 x 64]  = Q[128 x d] K_tile^T      tcgen05.mma, accumulator in TMEM
//   P = exp2(S - m)  (bf16, 128-byte-swizzled shared memory)
//   O[128 x d]  += P[128 x 64] V_tile       tcgen05.mma, accumulator in TMEM
// Roles: a producer warp streams K and V tiles (TMA, 128-byte swizzle, 3
// stages; blocks past the table or the pool load as zeros from out-of-range
// coordinates); one thread of the MMA warp issues the products and commits
// them to mbarriers; four softmax warps own one row each per thread (TMEM
// lane = row), read S with tcgen05.ld, mask (causal, sequence end), keep the
// running max and sum, write P, and rescale O in TMEM only when a row's max
// grows by more than 2^8 (otherwise the old max is kept: P stays <= 2^8).
// S is double-buffered in TMEM so that the next S product overlaps softmax.
// Every wait is bounded; on a timeout the kernel flags PKV_DEV_ERR_TIMEOUT,
// stops issuing, and still frees its TMEM.
#include "decode_common.cuh"

namespace pkv {

namespace {

using namespace dev;

constexpr int kRows = 128;                 // query rows per CTA (MMA M)
constexpr int kKeys = 64;                  // keys per tile (MMA N of S, K of P.V)
constexpr int kStages = 3;
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4, kMmaWarp = 5;
constexpr int kThreads = 6 * 32;
constexpr int kTmemCols = 256;             // S0 [0,64) S1 [64,128) O [128, 128 + d)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

__device__ __forceinline__ uint64_t umma_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    // start >> 4 [0,14), leading byte offset >> 4 [16,30), stride byte offset
    // >> 4 [32,46), version 1 [46,48), layout 128-byte swizzle (2) [61,64)
    return static_cast<uint64_t>((addr & 0x3FFFF) >> 4) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, A K-major,
// B K-major (b_mn = 0) or MN-major (b_mn = 1), N >> 3 at bit 17, M >> 4 at 24.
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(b_mn) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                     bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(static_cast<int>(accumulate))
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit TMEM columns: this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
        "%30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
        "%29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

template <int D>
struct TcGeometry {
    static constexpr int kHalves = D / 64;
    static constexpr int kQBytes = kHalves * kRows * 128;      // Q [half][row][128 B]
    static constexpr int kKVBytes = kHalves * kKeys * 128;     // K or V tile [half][key][128 B]
    static constexpr int kPBytes = kRows * 128;                // P [row][64 keys = 128 B]
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kQBytes;                    // + stage * kKVBytes
    static constexpr int kV = kK + kStages * kKVBytes;
    static constexpr int kP = kV + kStages * kKVBytes;
    static constexpr int kBars = kP + kPBytes;                 // 16 mbarriers
    static constexpr int kTmemSlot = kBars + 16 * 8;
    static constexpr int kSmemBytes = kTmemSlot + 16 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv, const PrefillParams p) {
    using Geo = TcGeometry<D>;
    const int b = blockIdx.z, kvh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;

    const int q0 = __ldg(p.query_start + b), q1 = __ldg(p.query_start + b + 1);
    const int ctx = __ldg(p.seq_lens + b);
    const int nq = q1 - q0;
    if (nq <= 0 || ctx < nq || ctx > p.W * kBlockTokens) {
        if (nq > 0 && blockIdx.x == 0 && kvh == 0 && threadIdx.x == 0) flag(p.err, PKV_DEV_ERR_BAD_LEN);
        return;
    }
    const int rows = nq * G;
    const int ntiles_q = (rows + kRows - 1) / kRows;
    if (static_cast<int>(blockIdx.x) >= ntiles_q) return;
    const int r_begin = (ntiles_q - 1 - static_cast<int>(blockIdx.x)) * kRows;  // heaviest first
    const int first_pos = ctx - nq;
    const int last_row = min(rows, r_begin + kRows) - 1;
    const int kv_end = first_pos + last_row / G + 1;        // keys this CTA can see
    const int nk = (kv_end + kKeys - 1) / kKeys;            // key tiles
    const int nblk_seq = (ctx + kBlockTokens - 1) / kBlockTokens;
    const long long oob_row = p.num_blocks * p.Hkv * kBlockTokens;  // past the tensor: zero fill

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t bar0 = smem_u32(smem + Geo::kBars);
    // barriers: kv_full[3] kv_empty[3] s_full[2] s_free[2] p_full o_done
    const auto kv_full = [&](int s) { return bar0 + 8 * s; };
    const auto kv_empty = [&](int s) { return bar0 + 8 * (3 + s); };
    const auto s_full = [&](int i) { return bar0 + 8 * (6 + i); };
    const auto s_free = [&](int i) { return bar0 + 8 * (8 + i); };
    const uint32_t p_full = bar0 + 8 * 10, o_done = bar0 + 8 * 11;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Geo::kTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Geo::kTmemSlot + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full(i), 1);
            mbar_init(s_free(i), kSoftmaxWarps);
        }
        mbar_init(p_full, kSoftmaxWarps);
        mbar_init(o_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "n"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // Q rows into shared memory (K-major, 128-byte swizzle): softmax thread t owns row t.
    int row_pos = -1;
    size_t out_off = 0;
    if (warp < kSoftmaxWarps) {
        const int t = threadIdx.x;
        const int r = r_begin + t;
        const uint4 *src = nullptr;
        if (r < rows) {
            const int tok = r / G, h = kvh * G + r % G;
            row_pos = first_pos + tok;
            out_off = (static_cast<size_t>(q0 + tok) * p.Hq + h) * D;
            src = reinterpret_cast<const uint4 *>(p.q + out_off);
        }
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            const uint4 v = src ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(smem + Geo::kQ + (c >> 3) * (kRows * 128) + t * 128 +
                                       (((c & 7) ^ (t & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_o = tmem + 128;

    if (warp == kProducerWarp) {
        if (lane == 0) {
            const uint64_t policy = l2_policy_evict_normal();
            const int32_t *trow = p.block_tables + static_cast<size_t>(b) * p.W;
            for (int j = 0; j < nk && !*abort_flag; ++j) {
                const int s = j % kStages;
                if (j >= kStages &&
                    !mbar_wait(kv_empty(s), static_cast<uint32_t>((j / kStages - 1) & 1), kWaitLimitNs)) {
                    flag(p.err, PKV_DEV_ERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(kv_full(s), 2 * Geo::kKVBytes);
                for (int i = 0; i < kKeys / kBlockTokens; ++i) {
                    const int blk = j * (kKeys / kBlockTokens) + i;
                    long long y = oob_row;  // blocks past the sequence or bad entries read as zeros
                    if (blk < nblk_seq) {
                        const int32_t phys = __ldg(trow + blk);
                        if (phys >= 0 && phys < p.num_blocks)
                            y = (static_cast<long long>(phys) * p.Hkv + kvh) * kBlockTokens;
                        else
                            flag(p.err, PKV_DEV_ERR_BAD_BLOCK);
                    }
#pragma unroll
                    for (int hh = 0; hh < Geo::kHalves; ++hh) {
                        const uint32_t off = hh * (kKeys * 128) + i * (kBlockTokens * 128);
                        tma_load_2d(smem_u32(smem + Geo::kK + s * Geo::kKVBytes) + off, &tmk, hh * 64,
                                    static_cast<int>(y), kv_full(s), policy);
                        tma_load_2d(smem_u32(smem + Geo::kV + s * Geo::kKVBytes) + off, &tmv, hh * 64,
                                    static_cast<int>(y), kv_full(s), policy);
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        constexpr uint32_t kIdS = umma_idesc(kRows, kKeys, 0);
        constexpr uint32_t kIdO = umma_idesc(kRows, D, 1);
        const auto issue_s = [&](int j) {  // S[j % 2] = Q . K_j^T
            const int s = j % kStages;
            const uint32_t kbase = smem_u32(smem + Geo::kK + s * Geo::kKVBytes);
            const uint32_t qbase = smem_u32(smem + Geo::kQ);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const int hh = k >> 2, kk = k & 3;
                umma(tmem + 64 * (j & 1), umma_desc(qbase + hh * (kRows * 128) + kk * 32, 16, 1024),
                     umma_desc(kbase + hh * (kKeys * 128) + kk * 32, 16, 1024), kIdS, k > 0);
            }
            umma_commit(s_full(j & 1));
        };
        bool ok = true;
        const auto wait = [&](uint32_t bar, uint32_t parity) {
            if (!ok) return;
            if (!mbar_wait(bar, parity, kWaitLimitNs)) {
                ok = false;
                if (lane == 0) {
                    flag(p.err, PKV_DEV_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
            }
        };
        wait(kv_full(0), 0);
        tc_fence_after();
        if (ok && lane == 0) issue_s(0);
        __syncwarp();
        for (int j = 0; j < nk && ok; ++j) {
            if (j + 1 < nk) {
                const int t = j + 1;
                wait(kv_full(t % kStages), static_cast<uint32_t>((t / kStages) & 1));
                if (t >= 2) wait(s_free(t & 1), static_cast<uint32_t>(((t - 2) / 2) & 1));
                tc_fence_after();
                if (ok && lane == 0) issue_s(t);
                __syncwarp();
            }
            // V rows of slots at or past the sequence end may hold anything: zero them
            const int s = j % kStages;
            const int k_lo = j * kKeys;
            if (ok && k_lo + kKeys > ctx && k_lo < nblk_seq * kBlockTokens) {
                const int z0 = max(ctx - k_lo, 0), z1 = min(nblk_seq * kBlockTokens - k_lo, kKeys);
                uint8_t *vbase = smem + Geo::kV + s * Geo::kKVBytes;
                for (int idx = lane; idx < (z1 - z0) * Geo::kHalves * 8; idx += 32) {
                    const int rr = z0 + idx / (Geo::kHalves * 8), rest = idx % (Geo::kHalves * 8);
                    *reinterpret_cast<uint4 *>(vbase + (rest >> 3) * (kKeys * 128) + rr * 128 +
                                               ((rest & 7) << 4)) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            wait(p_full, static_cast<uint32_t>(j & 1));
            tc_fence_after();
            if (ok && lane == 0) {
                const uint32_t pbase = smem_u32(smem + Geo::kP);
                const uint32_t vbase = smem_u32(smem + Geo::kV + s * Geo::kKVBytes);
#pragma unroll
                for (int k = 0; k < kKeys / 16; ++k)
                    umma(t_o, umma_desc(pbase + k * 32, 16, 1024),
                         umma_desc(vbase + k * (16 * 128), kKeys * 128, 1024), kIdO, j > 0 || k > 0);
                umma_commit(o_done);
                umma_commit(kv_empty(s));
            }
            __syncwarp();
        }
    } else {
        // ---------------- softmax warps: thread t = TMEM lane t = row r_begin + t
        const int t = threadIdx.x;
        const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < nk && ok; ++j) {
            if (!mbar_wait(s_full(j & 1), static_cast<uint32_t>((j >> 1) & 1), kWaitLimitNs) ||
                *abort_flag) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[2][32];
            tmem_ld32(tmem + lane_addr + 64 * (j & 1), sr[0]);
            tmem_ld32(tmem + lane_addr + 64 * (j & 1) + 32, sr[1]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_free(j & 1));
            // scores in the exp2 domain, causal mask by position
            float s[kKeys];
            float mx = -INFINITY;
            const int k0 = j * kKeys;
#pragma unroll
            for (int c = 0; c < kKeys; ++c) {
                const float v = __uint_as_float(sr[c >> 5][c & 31]) * p.scale_log2;
                s[c] = (k0 + c <= row_pos) ? v : -INFINITY;
                mx = fmaxf(mx, s[c]);
            }
            // keep the running max unless it grows by more than 2^8
            const bool grow = mx > m_run + kRescaleThreshold || (m_run == -INFINITY && mx != -INFINITY);
            const float m_new = grow ? mx : m_run;
            const float base = m_new == -INFINITY ? 0.f : m_new;
            float rowsum = 0.f;
            uint32_t pk[kKeys / 2];
#pragma unroll
            for (int c = 0; c < kKeys; c += 2) {
                const float a = exp2f(s[c] - base), bb = exp2f(s[c + 1] - base);
                rowsum += a + bb;
                __nv_bfloat162 h2 = __floats2bfloat162_rn(a, bb);
                pk[c / 2] = *reinterpret_cast<uint32_t *>(&h2);
            }
            // O and P belong to the previous product until it completes
            if (j > 0) {
                if (!mbar_wait(o_done, static_cast<uint32_t>((j - 1) & 1), kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float alpha = (grow && m_run != -INFINITY) ? exp2f(m_run - m_new) : 1.f;
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t o[32];
                        tmem_ld32(t_o + lane_addr + 32 * cc, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(t_o + lane_addr + 32 * cc, o);
                    }
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                }
                l_run *= alpha;
            }
            l_run += rowsum;
            m_run = m_new;
            // P row: 64 keys = 128 bytes, chunk c at c ^ (t & 7)
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(smem + Geo::kP + t * 128 + ((c ^ (t & 7)) << 4)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        if (ok && nk > 0 && mbar_wait(o_done, static_cast<uint32_t>((nk - 1) & 1), kWaitLimitNs)) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tmem_ld32(t_o + lane_addr + 32 * cc, o);
                if (row_pos >= 0) {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * inv,
                                                                  __uint_as_float(o[2 * i + 1]) * inv);
                        w[i] = *reinterpret_cast<uint32_t *>(&h2);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(p.out + out_off + 32 * cc);
#pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
        } else if (threadIdx.x == 0) {
            flag(p.err, PKV_DEV_ERR_TIMEOUT);
            *abort_flag = 1;
        }
    }
    // everyone (the producer's copies included) is done with TMEM and shared memory
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kTmemCols)
                     : "memory");
}

template <int D>
cudaError_t launch_prefill_tc_d(const CUtensorMap &tmk, const CUtensorMap &tmv,
                                const PrefillParams &p, int max_query_len, cudaStream_t stream) {
    constexpr int kSmem = TcGeometry<D>::kSmemBytes;
    auto kern = paged_prefill_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    const long long rows = static_cast<long long>(max_query_len) * p.group;
    const long long tiles = (rows + kRows - 1) / kRows;
    if (tiles == 0) return cudaSuccess;
    if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(p.Hkv), static_cast<unsigned>(p.B));
    kern<<<grid, kThreads, kSmem, stream>>>(tmk, tmv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const CUtensorMap &tmk, const CUtensorMap &tmv, const PrefillParams &p,
                              int head_dim, int max_query_len, cudaStream_t stream) {
    if (head_dim == 128) return launch_prefill_tc_d<128>(tmk, tmv, p, max_query_len, stream);
    if (head_dim == 64) return launch_prefill_tc_d<64>(tmk, tmv, p, max_query_len, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pkv
