/*
 * Paged decode attention oracle -- TEST INFRASTRUCTURE, not the product.
 *
 * A plain, slow fp64 CPU implementation of what the paged KV-cache hot path
 * computes.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg load it.  It shares no source, header, table or helper with the CUDA
 * library: it is written straight from the method's statement.
 *
 * Sources (page title, section):
 *  - "vLLM 與 PagedAttention：高吞吐推理的關鍵", section 二 "具體運作方式":
 *    the KV cache is cut into blocks of a fixed number of tokens (16), and a
 *    per-request block table maps logical block i to a physical block.
 *  - same page, section 三, step 三 (解碼): the new token's KV is written into
 *    the current block (a new block when it is full), then attention is
 *    computed over all earlier KV found through the block table.
 *  - "vLLM 与 PagedAttention：大模型高性能推理服务实战", section 三 3.2: 16
 *    tokens per block, logical token positions counted from 0.
 *
 * Readings where the pages are silent (all listed in the design notes):
 *  - attention is softmax(scale * q K^T) V over positions [0, len) of the
 *    sequence, len counting the token decoded this step;
 *  - grouped query heads: query head h reads KV head h / (Hq / Hkv);
 *  - cache layout [num_blocks][num_kv_heads][16][head_dim], K and V apart;
 *  - a slot is physical_block * 16 + offset; a negative slot means "skip";
 *  - len == 0 gives an all-zero output row.
 *
 * Every function is pinned by the CPU tests (worked examples from the pages,
 * closed forms, brute force against a library attention routine, invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BLOCK_TOKENS 16

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Element index of (block, kv_head, offset, dim) in one cache array. */
static size_t cache_index(int64_t block, int kv_head, int offset, int dim,
                          int num_kv_heads, int head_dim) {
    return (((size_t)block * (size_t)num_kv_heads + (size_t)kv_head) * ORACLE_BLOCK_TOKENS
            + (size_t)offset) * (size_t)head_dim + (size_t)dim;
}

/*
 * KV write, step 三 of the lifecycle: the new token's K and V go into the
 * slot the block manager handed out.  slot < 0: token skipped.
 * Returns 0, or -1 if a slot is outside the pool (nothing is written then).
 */
int oracle_kv_write(uint16_t *k_cache, uint16_t *v_cache,
                    const uint16_t *k, const uint16_t *v, const int64_t *slot_mapping,
                    int64_t num_tokens, int num_kv_heads, int head_dim, int64_t num_blocks) {
    for (int64_t t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= num_blocks * ORACLE_BLOCK_TOKENS) return -1;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t block = slot / ORACLE_BLOCK_TOKENS;
        int offset = (int)(slot % ORACLE_BLOCK_TOKENS);
        for (int h = 0; h < num_kv_heads; ++h)
            for (int e = 0; e < head_dim; ++e) {
                size_t src = ((size_t)t * num_kv_heads + h) * head_dim + e;
                size_t dst = cache_index(block, h, offset, e, num_kv_heads, head_dim);
                k_cache[dst] = k[src];
                v_cache[dst] = v[src];
            }
    }
    return 0;
}

/*
 * Copy-on-write block copy: a sequence that shares a partly filled block
 * (beam candidates share prefix blocks -- "vllm", PagedAttention 的核心原理)
 * gets a private copy before its next token is written.  Every slot of every
 * KV head of block src[i] is copied to block dst[i], pairs in order.
 * Returns 0, or -1 if an id is outside the pool (nothing copied then).
 */
int oracle_copy_blocks(uint16_t *k_cache, uint16_t *v_cache, const int64_t *src,
                       const int64_t *dst, int64_t n, int num_kv_heads, int head_dim,
                       int64_t num_blocks) {
    for (int64_t i = 0; i < n; ++i)
        if (src[i] < 0 || src[i] >= num_blocks || dst[i] < 0 || dst[i] >= num_blocks) return -1;
    for (int64_t i = 0; i < n; ++i)
        for (int h = 0; h < num_kv_heads; ++h)
            for (int off = 0; off < ORACLE_BLOCK_TOKENS; ++off)
                for (int e = 0; e < head_dim; ++e) {
                    size_t from = cache_index(src[i], h, off, e, num_kv_heads, head_dim);
                    size_t to = cache_index(dst[i], h, off, e, num_kv_heads, head_dim);
                    k_cache[to] = k_cache[from];
                    v_cache[to] = v_cache[from];
                }
    return 0;
}

/*
 * Swap space ("vLLM 与 PagedAttention：大模型高性能推理服务实战", section 二
 * 2.2, --swap-space: host memory for the KV of preempted requests).  Host
 * slots are laid out like cache blocks.  direction 0: GPU block gpu[i] ->
 * host slot host[i]; direction 1: the reverse.  Returns 0, or -1 on an id out
 * of range (nothing moved then).
 */
int oracle_swap_blocks(uint16_t *k_cache, uint16_t *v_cache, uint16_t *host_k, uint16_t *host_v,
                       const int64_t *gpu, const int64_t *host, int64_t n, int direction,
                       int num_kv_heads, int head_dim, int64_t num_blocks, int64_t num_host_blocks) {
    for (int64_t i = 0; i < n; ++i)
        if (gpu[i] < 0 || gpu[i] >= num_blocks || host[i] < 0 || host[i] >= num_host_blocks)
            return -1;
    for (int64_t i = 0; i < n; ++i)
        for (int h = 0; h < num_kv_heads; ++h)
            for (int off = 0; off < ORACLE_BLOCK_TOKENS; ++off)
                for (int e = 0; e < head_dim; ++e) {
                    size_t g = cache_index(gpu[i], h, off, e, num_kv_heads, head_dim);
                    size_t c = cache_index(host[i], h, off, e, num_kv_heads, head_dim);
                    if (direction == 0) {
                        host_k[c] = k_cache[g];
                        host_v[c] = v_cache[g];
                    } else {
                        k_cache[g] = host_k[c];
                        v_cache[g] = host_v[c];
                    }
                }
    return 0;
}

/*
 * Copy the logical K and V rows of one sequence and KV head, in token order,
 * through the block table (section 二: logical block p/16 -> physical block).
 * Returns -1 if a table entry on the path is outside [0, num_blocks).
 */
static int gather_sequence(double *K, double *V, const uint16_t *k_cache, const uint16_t *v_cache,
                           const int32_t *table_row, int len, int kv_head,
                           int num_kv_heads, int head_dim, int64_t num_blocks) {
    for (int p = 0; p < len; ++p) {
        int32_t phys = table_row[p / ORACLE_BLOCK_TOKENS];
        if (phys < 0 || (int64_t)phys >= num_blocks) return -1;
        int offset = p % ORACLE_BLOCK_TOKENS;
        for (int e = 0; e < head_dim; ++e) {
            size_t idx = cache_index(phys, kv_head, offset, e, num_kv_heads, head_dim);
            K[(size_t)p * head_dim + e] = bf16_bits_to_double(k_cache[idx]);
            V[(size_t)p * head_dim + e] = bf16_bits_to_double(v_cache[idx]);
        }
    }
    return 0;
}

/* out[e] = sum_p softmax(scale * q.K[p])_p * V[p][e], the max subtracted first. */
static void attend(double *out, const double *qv, const double *K, const double *V,
                   int len, int head_dim, double scale, double *s) {
    for (int e = 0; e < head_dim; ++e) out[e] = 0.0;
    if (len == 0) return;
    double m = -INFINITY;
    for (int p = 0; p < len; ++p) {
        double acc = 0.0;
        for (int e = 0; e < head_dim; ++e) acc += qv[e] * K[(size_t)p * head_dim + e];
        s[p] = scale * acc;
        if (s[p] > m) m = s[p];
    }
    double z = 0.0;
    for (int p = 0; p < len; ++p) {
        s[p] = exp(s[p] - m);
        z += s[p];
    }
    for (int p = 0; p < len; ++p)
        for (int e = 0; e < head_dim; ++e) out[e] += s[p] * V[(size_t)p * head_dim + e];
    for (int e = 0; e < head_dim; ++e) out[e] /= z;
}

/*
 * Decode attention for every (sequence, query head): out [B][Hq][d] fp64.
 * q [B][Hq][d], caches [NB][Hkv][16][d] as bf16 bits; block_tables [B][W].
 * nthreads <= 0 uses the OpenMP default.  Returns 0, -1 on a bad table entry,
 * -2 on bad sizes, -3 when out of memory.
 */
int oracle_paged_decode(double *out, const uint16_t *q,
                        const uint16_t *k_cache, const uint16_t *v_cache,
                        const int32_t *block_tables, int width, const int32_t *seq_lens,
                        int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                        int64_t num_blocks, double scale, int nthreads) {
    if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads) return -2;
    for (int b = 0; b < num_seqs; ++b)
        if (seq_lens[b] < 0 || seq_lens[b] > width * ORACLE_BLOCK_TOKENS) return -2;
    const int group = num_heads / num_kv_heads;
    int status = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int item = 0; item < num_seqs * num_kv_heads; ++item) {
        int b = item / num_kv_heads, kvh = item % num_kv_heads;
        int len = seq_lens[b];
        size_t n = (size_t)(len > 0 ? len : 1) * head_dim;
        double *K = malloc(n * sizeof *K), *V = malloc(n * sizeof *V);
        double *s = malloc((size_t)(len > 0 ? len : 1) * sizeof *s);
        double *qv = malloc((size_t)head_dim * sizeof *qv);
        if (!K || !V || !s || !qv) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = -3;
        } else if (gather_sequence(K, V, k_cache, v_cache, block_tables + (size_t)b * width, len,
                                   kvh, num_kv_heads, head_dim, num_blocks)) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = -1;
        } else {
            for (int h = kvh * group; h < (kvh + 1) * group; ++h) {
                for (int e = 0; e < head_dim; ++e)
                    qv[e] = bf16_bits_to_double(q[((size_t)b * num_heads + h) * head_dim + e]);
                attend(out + ((size_t)b * num_heads + h) * head_dim, qv, K, V, len, head_dim,
                       scale, s);
            }
        }
        free(K); free(V); free(s); free(qv);
    }
    return status;
}

/*
 * The same result computed in partitions of `partition_tokens` positions.
 * Each partition gives its own max m_p, sum l_p = sum exp(s - m_p) and
 * unnormalised o_p = sum exp(s - m_p) V; the partitions are then combined
 * with M = max m_p:  out = sum_p e^{m_p - M} o_p / sum_p e^{m_p - M} l_p.
 * Exactly equal to oracle_paged_decode in real arithmetic (it is how a
 * long context is cut into independent pieces); used to check that identity.
 */
int oracle_paged_decode_partitioned(double *out, const uint16_t *q,
                                    const uint16_t *k_cache, const uint16_t *v_cache,
                                    const int32_t *block_tables, int width, const int32_t *seq_lens,
                                    int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                    int64_t num_blocks, double scale, int partition_tokens) {
    if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads || partition_tokens <= 0)
        return -2;
    const int group = num_heads / num_kv_heads;
    for (int b = 0; b < num_seqs; ++b) {
        int len = seq_lens[b];
        if (len < 0 || len > width * ORACLE_BLOCK_TOKENS) return -2;
        size_t n = (size_t)(len > 0 ? len : 1) * head_dim;
        double *K = malloc(n * sizeof *K), *V = malloc(n * sizeof *V);
        double *o = malloc((size_t)head_dim * sizeof *o);
        if (!K || !V || !o) { free(K); free(V); free(o); return -3; }
        for (int kvh = 0; kvh < num_kv_heads; ++kvh) {
            if (gather_sequence(K, V, k_cache, v_cache, block_tables + (size_t)b * width, len, kvh,
                                num_kv_heads, head_dim, num_blocks)) {
                free(K); free(V); free(o);
                return -1;
            }
            for (int h = kvh * group; h < (kvh + 1) * group; ++h) {
                const uint16_t *qh = q + ((size_t)b * num_heads + h) * head_dim;
                double *dst = out + ((size_t)b * num_heads + h) * head_dim;
                int nparts = (len + partition_tokens - 1) / partition_tokens;
                double M = -INFINITY;
                for (int part = 0; part < nparts; ++part)
                    for (int p = part * partition_tokens; p < len && p < (part + 1) * partition_tokens; ++p) {
                        double acc = 0.0;
                        for (int e = 0; e < head_dim; ++e)
                            acc += bf16_bits_to_double(qh[e]) * K[(size_t)p * head_dim + e];
                        if (scale * acc > M) M = scale * acc;
                    }
                double L = 0.0;
                for (int e = 0; e < head_dim; ++e) dst[e] = 0.0;
                for (int part = 0; part < nparts; ++part) {
                    int lo = part * partition_tokens;
                    int hi = lo + partition_tokens < len ? lo + partition_tokens : len;
                    double m_p = -INFINITY, l_p = 0.0;
                    for (int p = lo; p < hi; ++p) {
                        double acc = 0.0;
                        for (int e = 0; e < head_dim; ++e)
                            acc += bf16_bits_to_double(qh[e]) * K[(size_t)p * head_dim + e];
                        if (scale * acc > m_p) m_p = scale * acc;
                    }
                    for (int e = 0; e < head_dim; ++e) o[e] = 0.0;
                    for (int p = lo; p < hi; ++p) {
                        double acc = 0.0;
                        for (int e = 0; e < head_dim; ++e)
                            acc += bf16_bits_to_double(qh[e]) * K[(size_t)p * head_dim + e];
                        double w = exp(scale * acc - m_p);
                        l_p += w;
                        for (int e = 0; e < head_dim; ++e) o[e] += w * V[(size_t)p * head_dim + e];
                    }
                    double c = exp(m_p - M);
                    L += c * l_p;
                    for (int e = 0; e < head_dim; ++e) dst[e] += c * o[e];
                }
                if (nparts > 0)
                    for (int e = 0; e < head_dim; ++e) dst[e] /= L;
            }
        }
        free(K); free(V); free(o);
    }
    return 0;
}

int oracle_block_tokens(void) { return ORACLE_BLOCK_TOKENS; }
