// Device building blocks shared by the decode kernels: the swizzled tile
// addressing, the block-table read-ahead window and the per-warp attention
// state of the CUDA-core (one query row per KV head) and tensor-core (group
// of query heads) paths.  See decode.cu for the method and the layouts.
#pragma once

#include <cfloat>
#include <type_traits>

#include "../../include/pkv.h"
#include "internal.h"
#include "ptx.cuh"

namespace pkv {

// Launches `kern` so that it may be scheduled before the preceding kernel in
// the stream finishes (programmatic dependent launch); the kernel must call
// pdl_wait_primary() before it touches memory that kernel may use.  Every
// kernel of the decode path is launched this way and waits before its first
// access to such memory (the host-written lengths and tables may be read
// earlier), so that a call's grid is scheduled while the previous call's
// last grid drains (that grid lets its dependents launch once all its CTAs
// have started).
template <typename... Args>
cudaError_t launch_dependent_smem(void (*kern)(Args...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename... Args>
cudaError_t launch_dependent(void (*kern)(Args...), dim3 grid, dim3 block, cudaStream_t stream,
                             Args... args) {
    return launch_dependent_smem(kern, grid, block, 0, stream, args...);
}

namespace dev {

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

    // Sums o over the row groups (complete in lanes < CH, chunk c = lane) and
    // l over the warp (complete in every lane).
    __device__ __forceinline__ void reduce() {
#pragma unroll
        for (int m = CH; m < 32; m <<= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] += __shfl_xor_sync(0xffffffffu, o[e], m);
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, m);
    }

    // Writes this warp's (m, l, o[D]) into red (D + 2 floats).
    __device__ __forceinline__ void finish(float *red, int lane) {
        reduce();
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

    // Sums l over the 8 lanes that share a pair of heads.
    __device__ __forceinline__ void reduce() {
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
            l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], m);
            l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], m);
        }
    }

    // Writes this warp's m[8], l[8], o[8][D] into red (16 + 8 * D floats).
    __device__ __forceinline__ void finish(float *red, int lane) {
        const int tig = lane & 3, gid = lane >> 2;
        reduce();
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

}  // namespace dev
}  // namespace pkv
