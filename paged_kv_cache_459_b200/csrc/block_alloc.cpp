// Host block allocator: reference-counted physical blocks, per-sequence block
// tables, on-demand allocation, prefix sharing and release.
//
// Follows "vLLM 與 PagedAttention：高吞吐推理的關鍵": section 二 (fixed 16-token
// blocks; a table maps logical block i to a physical block; several tables may
// point at the same blocks) and section 三 (an empty table at admission, a new
// block whenever the current one fills during prefill and decode, every block
// returned when the request finishes).  Reference counts reconcile sharing
// with release: a block goes back to the pool when its last holder lets go.
//
// The free list is a first-in first-out queue: blocks are taken from the
// front and returned to the back, starting from a caller-given permutation, so
// tables are reproducible for a seed.  Every call validates first and mutates
// only once it cannot fail, so an error leaves the state unchanged; the free
// lists are rings sized once for the whole pool, so returning blocks never
// allocates.
#include <algorithm>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pkv.h"

namespace {

constexpr int64_t kBlockTokens = PKV_BLOCK_TOKENS;

int64_t blocks_for(int64_t tokens) { return (tokens + kBlockTokens - 1) / kBlockTokens; }

struct Sequence {
    std::vector<int32_t> blocks;  // GPU blocks, or host slots while swapped out
    int64_t len = 0;
    bool swapped = false;
    uint64_t mark = 0;  // the batch call that last named it (duplicate check)
};

// What appending one token to a sequence takes: room in its last block, a
// fresh block (none yet, or the last one is full), or a copy-on-write of a
// partly filled last block that other tables also hold.
enum class AppendKind : uint8_t { kInPlace, kNewBlock, kCopyOnWrite };

// Fixed-capacity FIFO of block (or host slot) ids.  A pool never has more
// free entries than entries, so the ring is sized once (init, which may
// throw) and push_back never allocates.
class BlockFifo {
public:
    void init(size_t capacity) {
        buf_.assign(std::max<size_t>(capacity, 1), 0);
        head_ = size_ = 0;
    }
    size_t size() const { return size_; }
    bool empty() const { return size_ == 0; }
    int32_t front() const { return buf_[head_]; }
    int32_t operator[](size_t i) const { return buf_[(head_ + i) % buf_.size()]; }
    void pop_front() {
        head_ = (head_ + 1) % buf_.size();
        --size_;
    }
    void push_back(int32_t v) {  // the caller keeps size() below the capacity
        buf_[(head_ + size_) % buf_.size()] = v;
        ++size_;
    }

private:
    std::vector<int32_t> buf_;
    size_t head_ = 0, size_ = 0;
};

}  // namespace

struct pkv_alloc {
    int64_t num_blocks = 0;
    BlockFifo free_list;  // capacity num_blocks
    std::vector<int32_t> refcount;
    std::unordered_map<int64_t, Sequence> seqs;
    // Copy-on-write block copies (src, dst) not yet taken by the caller.
    std::vector<std::pair<int32_t, int32_t>> pending_copies;
    // Host swap space: free host block slots, and queued moves (GPU block,
    // host slot) out of and into the GPU pool.
    BlockFifo host_free;  // capacity num_host_blocks
    int64_t num_host_blocks = 0;
    std::vector<std::pair<int32_t, int32_t>> pending_out, pending_in;
    // Scratch of the batch append, kept between calls (no allocation per step).
    uint64_t epoch = 0;
    std::vector<Sequence *> batch_seqs;
    std::vector<AppendKind> batch_kinds;
};

static pkv_status prefix_groups(const pkv_alloc *a, const int64_t *seq_ids, int n,
                                int32_t *prefix_blocks_out, int32_t *group_offsets_out,
                                int32_t *group_seqs_out, int32_t *num_groups_out);

extern "C" {

pkv_status pkv_alloc_create(int64_t num_blocks, const int64_t *free_order, pkv_alloc **out) {
    if (!out || num_blocks <= 0 || num_blocks > INT32_MAX) return PKV_ERR_INVALID_ARG;
    *out = nullptr;
    pkv_alloc *a = new (std::nothrow) pkv_alloc;
    if (!a) return PKV_ERR_OOM;
    try {
        a->num_blocks = num_blocks;
        a->refcount.assign(static_cast<size_t>(num_blocks), 0);
        a->free_list.init(static_cast<size_t>(num_blocks));
        a->host_free.init(0);
        if (free_order) {
            std::vector<char> seen(static_cast<size_t>(num_blocks), 0);
            for (int64_t i = 0; i < num_blocks; ++i) {
                int64_t b = free_order[i];
                if (b < 0 || b >= num_blocks || seen[b]) {
                    delete a;
                    return PKV_ERR_INVALID_ARG;
                }
                seen[b] = 1;
                a->free_list.push_back(static_cast<int32_t>(b));
            }
        } else {
            for (int64_t i = 0; i < num_blocks; ++i) a->free_list.push_back(static_cast<int32_t>(i));
        }
    } catch (const std::bad_alloc &) {
        delete a;
        return PKV_ERR_OOM;
    }
    *out = a;
    return PKV_OK;
}

void pkv_alloc_destroy(pkv_alloc *a) { delete a; }

pkv_status pkv_alloc_add_seq(pkv_alloc *a, int64_t seq_id, int64_t num_tokens) {
    if (!a || num_tokens < 0 || a->seqs.count(seq_id)) return PKV_ERR_INVALID_ARG;
    int64_t need = blocks_for(num_tokens);
    if (need > static_cast<int64_t>(a->free_list.size())) return PKV_ERR_OOM;
    try {
        Sequence s;
        s.blocks.reserve(static_cast<size_t>(need));
        s.len = num_tokens;
        for (int64_t i = 0; i < need; ++i) s.blocks.push_back(a->free_list[static_cast<size_t>(i)]);
        a->seqs.emplace(seq_id, std::move(s));
    } catch (const std::bad_alloc &) {
        return PKV_ERR_OOM;
    }
    for (int64_t i = 0; i < need; ++i) {
        a->refcount[a->free_list.front()] = 1;
        a->free_list.pop_front();
    }
    return PKV_OK;
}

pkv_status pkv_alloc_fork(pkv_alloc *a, int64_t parent, int64_t child, int64_t num_tokens) {
    if (!a) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(parent);
    if (it == a->seqs.end() || it->second.swapped || a->seqs.count(child)) return PKV_ERR_INVALID_ARG;
    int64_t n = num_tokens < 0 ? it->second.len : num_tokens;
    if (n > it->second.len) return PKV_ERR_INVALID_ARG;
    Sequence *made = nullptr;
    try {
        Sequence s;
        s.len = n;
        s.blocks.assign(it->second.blocks.begin(), it->second.blocks.begin() + blocks_for(n));
        made = &a->seqs.emplace(child, std::move(s)).first->second;  // may rehash: `it` is stale after
    } catch (const std::bad_alloc &) {
        return PKV_ERR_OOM;
    }
    for (int32_t b : made->blocks) a->refcount[b] += 1;  // only once the child exists
    return PKV_OK;
}

static AppendKind append_kind(const Sequence &s, int32_t last_refcount) {
    if (s.len % kBlockTokens == 0) return AppendKind::kNewBlock;
    return last_refcount > 1 ? AppendKind::kCopyOnWrite : AppendKind::kInPlace;
}

static int64_t do_append(pkv_alloc *a, Sequence &s, AppendKind kind) {
    if (kind != AppendKind::kInPlace) {
        int32_t b = a->free_list.front();
        a->free_list.pop_front();
        a->refcount[b] = 1;
        if (kind == AppendKind::kNewBlock) {
            s.blocks.push_back(b);
        } else {  // the sequence gets a private copy of its shared last block
            const int32_t old = s.blocks.back();
            a->refcount[old] -= 1;  // still >= 1: other tables hold it
            a->pending_copies.emplace_back(old, b);
            s.blocks.back() = b;
        }
    }
    int64_t pos = s.len++;
    return static_cast<int64_t>(s.blocks[pos / kBlockTokens]) * kBlockTokens + pos % kBlockTokens;
}

pkv_status pkv_alloc_append_token(pkv_alloc *a, int64_t seq_id, int64_t *slot_out) {
    if (!a || !slot_out) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || it->second.swapped) return PKV_ERR_INVALID_ARG;
    Sequence &s = it->second;
    const AppendKind kind = append_kind(s, s.blocks.empty() ? 0 : a->refcount[s.blocks.back()]);
    if (kind != AppendKind::kInPlace && a->free_list.empty()) return PKV_ERR_OOM;
    try {
        if (kind == AppendKind::kNewBlock) s.blocks.reserve(s.blocks.size() + 1);
        if (kind == AppendKind::kCopyOnWrite) a->pending_copies.reserve(a->pending_copies.size() + 1);
    } catch (const std::bad_alloc &) {
        return PKV_ERR_OOM;
    }
    *slot_out = do_append(a, s, kind);
    return PKV_OK;
}

// One token for each of n distinct sequences, all or none.  With a table
// (width > 0), every sequence must keep its blocks within width, and row i of
// tables_io / lens_io[i] get the entry and length the append changed.
static pkv_status append_batch(pkv_alloc *a, const int64_t *seq_ids, int n, int64_t *slots_out,
                               int width, int32_t *tables_io, int32_t *lens_io) {
    std::vector<Sequence *> &seqs = a->batch_seqs;
    std::vector<AppendKind> &kinds = a->batch_kinds;
    seqs.clear();
    kinds.clear();
    // a sequence named twice in one call is an error: each sequence carries
    // the number of the last call that named it
    const uint64_t epoch = ++a->epoch;
    try {
        std::unordered_map<int32_t, int32_t> released;  // copy-on-writes earlier in this batch
        seqs.reserve(static_cast<size_t>(n));
        kinds.reserve(static_cast<size_t>(n));
        int64_t new_blocks = 0, cows = 0;
        for (int i = 0; i < n; ++i) {
            auto it = a->seqs.find(seq_ids[i]);
            if (it == a->seqs.end() || it->second.swapped) return PKV_ERR_INVALID_ARG;
            Sequence &s = it->second;
            if (s.mark == epoch) return PKV_ERR_INVALID_ARG;
            s.mark = epoch;
            int32_t rc = 0;
            if (!s.blocks.empty()) {
                rc = a->refcount[s.blocks.back()];
                if (!released.empty()) {
                    auto r = released.find(s.blocks.back());
                    if (r != released.end()) rc -= r->second;
                }
            }
            const AppendKind kind = append_kind(s, rc);
            if (tables_io && (s.len >= INT32_MAX ||
                              static_cast<int64_t>(s.blocks.size()) + (kind == AppendKind::kNewBlock) > width))
                return PKV_ERR_INVALID_ARG;
            if (kind == AppendKind::kNewBlock) s.blocks.reserve(s.blocks.size() + 1);
            if (kind == AppendKind::kCopyOnWrite) {
                released[s.blocks.back()] += 1;
                ++cows;
            }
            new_blocks += kind != AppendKind::kInPlace;
            seqs.push_back(&s);
            kinds.push_back(kind);
        }
        if (new_blocks > static_cast<int64_t>(a->free_list.size())) return PKV_ERR_OOM;
        a->pending_copies.reserve(a->pending_copies.size() + static_cast<size_t>(cows));
    } catch (const std::bad_alloc &) {
        return PKV_ERR_OOM;
    }
    for (int i = 0; i < n; ++i) slots_out[i] = do_append(a, *seqs[i], kinds[i]);
    if (tables_io) {
        for (int i = 0; i < n; ++i) {
            const Sequence &s = *seqs[i];
            // the last entry is the only one an append changes (a new block, or
            // the private copy that replaces a shared one)
            tables_io[static_cast<size_t>(i) * width + s.blocks.size() - 1] = s.blocks.back();
            lens_io[i] = static_cast<int32_t>(s.len);
        }
    }
    return PKV_OK;
}

pkv_status pkv_alloc_append_tokens(pkv_alloc *a, const int64_t *seq_ids, int n, int64_t *slots_out) {
    if (!a || n < 0 || (n > 0 && (!seq_ids || !slots_out))) return PKV_ERR_INVALID_ARG;
    return append_batch(a, seq_ids, n, slots_out, 0, nullptr, nullptr);
}

pkv_status pkv_alloc_append_tokens_into(pkv_alloc *a, const int64_t *seq_ids, int n, int64_t *slots_out,
                                        int width, int32_t *tables_io, int32_t *lens_io) {
    if (!a || n < 0 || width <= 0 || (n > 0 && (!seq_ids || !slots_out || !tables_io || !lens_io)))
        return PKV_ERR_INVALID_ARG;
    return append_batch(a, seq_ids, n, slots_out, width, tables_io, lens_io);
}

pkv_status pkv_alloc_extend(pkv_alloc *a, int64_t seq_id, int64_t n, int64_t *slots_out) {
    if (!a || n < 0 || (n > 0 && !slots_out)) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || it->second.swapped) return PKV_ERR_INVALID_ARG;
    Sequence &s = it->second;
    if (n == 0) return PKV_OK;
    // blocks needed: a private copy of a shared partly filled last block, then
    // one per 16 positions past the current blocks
    const bool cow = s.len % kBlockTokens != 0 && a->refcount[s.blocks.back()] > 1;
    const int64_t need = (cow ? 1 : 0) + blocks_for(s.len + n) - static_cast<int64_t>(s.blocks.size());
    if (need > static_cast<int64_t>(a->free_list.size())) return PKV_ERR_OOM;
    try {
        s.blocks.reserve(static_cast<size_t>(blocks_for(s.len + n)));
        if (cow) a->pending_copies.reserve(a->pending_copies.size() + 1);
    } catch (const std::bad_alloc &) {
        return PKV_ERR_OOM;
    }
    for (int64_t i = 0; i < n; ++i)
        slots_out[i] = do_append(a, s, append_kind(s, s.blocks.empty() ? 0 : a->refcount[s.blocks.back()]));
    return PKV_OK;
}

pkv_status pkv_alloc_take_copies(pkv_alloc *a, int64_t *src_out, int64_t *dst_out, int64_t cap,
                                 int64_t *n_out) {
    if (!a || !n_out || cap < 0 || (cap > 0 && (!src_out || !dst_out))) return PKV_ERR_INVALID_ARG;
    const int64_t n = static_cast<int64_t>(a->pending_copies.size());
    *n_out = n;
    if (cap < n) return PKV_OK;  // nothing taken: ask again with room for all
    for (int64_t i = 0; i < n; ++i) {
        src_out[i] = a->pending_copies[static_cast<size_t>(i)].first;
        dst_out[i] = a->pending_copies[static_cast<size_t>(i)].second;
    }
    a->pending_copies.clear();
    return PKV_OK;
}

pkv_status pkv_alloc_free_seq(pkv_alloc *a, int64_t seq_id) {
    if (!a) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
    if (it->second.swapped) {
        for (int32_t h : it->second.blocks) a->host_free.push_back(h);
    } else {
        for (int32_t b : it->second.blocks) {
            if (--a->refcount[b] == 0) a->free_list.push_back(b);
        }
    }
    a->seqs.erase(it);
    return PKV_OK;
}

pkv_status pkv_alloc_set_host_pool(pkv_alloc *a, int64_t num_host_blocks) {
    if (!a || num_host_blocks < 0 || num_host_blocks > INT32_MAX) return PKV_ERR_INVALID_ARG;
    for (const auto &kv : a->seqs)
        if (kv.second.swapped) return PKV_ERR_INVALID_ARG;  // host slots in use
    try {
        BlockFifo fresh;
        fresh.init(static_cast<size_t>(num_host_blocks));
        for (int64_t i = 0; i < num_host_blocks; ++i) fresh.push_back(static_cast<int32_t>(i));
        a->host_free = std::move(fresh);
    } catch (const std::bad_alloc &) {
        return PKV_ERR_OOM;
    }
    a->num_host_blocks = num_host_blocks;
    return PKV_OK;
}

pkv_status pkv_alloc_swap_out(pkv_alloc *a, int64_t seq_id) {
    if (!a) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || it->second.swapped) return PKV_ERR_INVALID_ARG;
    Sequence &s = it->second;
    for (int32_t b : s.blocks)
        if (a->refcount[b] != 1) return PKV_ERR_UNSUPPORTED;  // shared blocks stay on the GPU
    if (s.blocks.size() > a->host_free.size()) return PKV_ERR_OOM;
    try {
        a->pending_out.reserve(a->pending_out.size() + s.blocks.size());
    } catch (const std::bad_alloc &) {
        return PKV_ERR_OOM;
    }
    for (int32_t &b : s.blocks) {
        const int32_t h = a->host_free.front();
        a->host_free.pop_front();
        a->pending_out.emplace_back(b, h);
        a->refcount[b] = 0;
        a->free_list.push_back(b);
        b = h;
    }
    s.swapped = true;
    return PKV_OK;
}

pkv_status pkv_alloc_swap_in(pkv_alloc *a, int64_t seq_id) {
    if (!a) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || !it->second.swapped) return PKV_ERR_INVALID_ARG;
    Sequence &s = it->second;
    if (s.blocks.size() > a->free_list.size()) return PKV_ERR_OOM;
    try {
        a->pending_in.reserve(a->pending_in.size() + s.blocks.size());
    } catch (const std::bad_alloc &) {
        return PKV_ERR_OOM;
    }
    for (int32_t &h : s.blocks) {
        const int32_t b = a->free_list.front();
        a->free_list.pop_front();
        a->refcount[b] = 1;
        a->pending_in.emplace_back(b, h);
        a->host_free.push_back(h);
        h = b;
    }
    s.swapped = false;
    return PKV_OK;
}

static pkv_status take_pairs(std::vector<std::pair<int32_t, int32_t>> &q, int64_t *gpu_out,
                             int64_t *host_out, int64_t cap, int64_t *n_out) {
    if (!n_out || cap < 0 || (cap > 0 && (!gpu_out || !host_out))) return PKV_ERR_INVALID_ARG;
    const int64_t n = static_cast<int64_t>(q.size());
    *n_out = n;
    if (cap < n) return PKV_OK;
    for (int64_t i = 0; i < n; ++i) {
        gpu_out[i] = q[static_cast<size_t>(i)].first;
        host_out[i] = q[static_cast<size_t>(i)].second;
    }
    q.clear();
    return PKV_OK;
}

pkv_status pkv_alloc_take_swaps(pkv_alloc *a, int direction, int64_t *gpu_out, int64_t *host_out,
                                int64_t cap, int64_t *n_out) {
    if (!a || (direction != PKV_SWAP_OUT && direction != PKV_SWAP_IN)) return PKV_ERR_INVALID_ARG;
    return take_pairs(direction == PKV_SWAP_OUT ? a->pending_out : a->pending_in, gpu_out, host_out,
                      cap, n_out);
}

pkv_status pkv_alloc_export(const pkv_alloc *a, const int64_t *seq_ids, int n, int width,
                            int32_t *tables_out, int32_t *lens_out) {
    if (!a || n < 0 || width <= 0 || (n > 0 && (!seq_ids || !tables_out || !lens_out)))
        return PKV_ERR_INVALID_ARG;
    // every sequence checked before any row is written, each looked up once
    // (the lookups of up to kStack sequences kept on the stack)
    constexpr int kStack = 256;
    const Sequence *stack_buf[kStack];
    std::vector<const Sequence *> heap_buf;
    const Sequence **found = stack_buf;
    if (n > kStack) {
        try {
            heap_buf.resize(static_cast<size_t>(n));
        } catch (const std::bad_alloc &) {
            return PKV_ERR_OOM;
        }
        found = heap_buf.data();
    }
    for (int i = 0; i < n; ++i) {
        auto it = a->seqs.find(seq_ids[i]);
        if (it == a->seqs.end() || it->second.swapped) return PKV_ERR_INVALID_ARG;
        if (static_cast<int64_t>(it->second.blocks.size()) > width || it->second.len > INT32_MAX)
            return PKV_ERR_INVALID_ARG;
        found[i] = &it->second;
    }
    for (int i = 0; i < n; ++i) {
        const Sequence &s = *found[i];
        int32_t *row = tables_out + static_cast<size_t>(i) * width;
        std::copy(s.blocks.begin(), s.blocks.end(), row);
        std::fill(row + s.blocks.size(), row + width, -1);
        lens_out[i] = static_cast<int32_t>(s.len);
    }
    return PKV_OK;
}

pkv_status pkv_alloc_stats(const pkv_alloc *a, int64_t *free_blocks, int64_t *used_blocks,
                           int64_t *shared_blocks, double *utilisation) {
    if (!a) return PKV_ERR_INVALID_ARG;
    int64_t free_n = static_cast<int64_t>(a->free_list.size());
    int64_t used = a->num_blocks - free_n;
    int64_t shared = 0;
    for (int32_t r : a->refcount) shared += r > 1;
    double util = 0.0;
    if (used > 0) {
        std::vector<int16_t> fill;
        try {
            fill.assign(static_cast<size_t>(a->num_blocks), 0);
        } catch (const std::bad_alloc &) {
            return PKV_ERR_OOM;
        }
        for (const auto &kv : a->seqs) {
            const Sequence &s = kv.second;
            if (s.swapped) continue;
            for (size_t j = 0; j < s.blocks.size(); ++j) {
                int64_t f = std::min<int64_t>(kBlockTokens, s.len - static_cast<int64_t>(j) * kBlockTokens);
                int16_t &slot = fill[s.blocks[j]];
                slot = std::max<int16_t>(slot, static_cast<int16_t>(f));
            }
        }
        int64_t filled = 0;
        for (int16_t f : fill) filled += f;
        util = static_cast<double>(filled) / static_cast<double>(kBlockTokens * used);
    }
    if (free_blocks) *free_blocks = free_n;
    if (used_blocks) *used_blocks = used;
    if (shared_blocks) *shared_blocks = shared;
    if (utilisation) *utilisation = util;
    return PKV_OK;
}

pkv_status pkv_alloc_free_list(const pkv_alloc *a, int64_t *out, int64_t cap, int64_t *n_out) {
    if (!a || !n_out || cap < 0 || (cap > 0 && !out)) return PKV_ERR_INVALID_ARG;
    int64_t n = static_cast<int64_t>(a->free_list.size());
    int64_t m = std::min(n, cap);
    for (int64_t i = 0; i < m; ++i) out[i] = a->free_list[static_cast<size_t>(i)];
    *n_out = n;
    return PKV_OK;
}

pkv_status pkv_alloc_prefix_groups(const pkv_alloc *a, const int64_t *seq_ids, int n,
                                   int32_t *prefix_blocks_out, int32_t *group_offsets_out,
                                   int32_t *group_seqs_out, int32_t *num_groups_out) {
    if (!a || n < 0 || !num_groups_out ||
        (n > 0 && (!seq_ids || !prefix_blocks_out || !group_offsets_out || !group_seqs_out)))
        return PKV_ERR_INVALID_ARG;
    try {
        return prefix_groups(a, seq_ids, n, prefix_blocks_out, group_offsets_out, group_seqs_out,
                             num_groups_out);
    } catch (const std::bad_alloc &) {  // before any output is written
        return PKV_ERR_OOM;
    }
}

}  // extern "C"

static pkv_status prefix_groups(const pkv_alloc *a, const int64_t *seq_ids, int n,
                                int32_t *prefix_blocks_out, int32_t *group_offsets_out,
                                int32_t *group_seqs_out, int32_t *num_groups_out) {
    std::vector<const Sequence *> seqs(static_cast<size_t>(n));
    for (int i = 0; i < n; ++i) {
        auto it = a->seqs.find(seq_ids[i]);
        if (it == a->seqs.end() || it->second.swapped) return PKV_ERR_INVALID_ARG;
        seqs[i] = &it->second;
    }
    // Candidates: sequences whose first block is full and held by several tables,
    // grouped by that block in order of first appearance.
    std::vector<int> order;  // distinct first blocks, first appearance order
    std::unordered_map<int32_t, std::vector<int>> by_first;
    for (int i = 0; i < n; ++i) {
        const Sequence &s = *seqs[i];
        if (s.len < kBlockTokens || a->refcount[s.blocks[0]] < 2) continue;
        auto &v = by_first[s.blocks[0]];
        if (v.empty()) order.push_back(s.blocks[0]);
        v.push_back(i);
    }
    std::fill(prefix_blocks_out, prefix_blocks_out + n, 0);
    int32_t groups = 0, pos = 0;
    group_offsets_out[0] = 0;
    for (int32_t blk : order) {
        const std::vector<int> &members = by_first[blk];
        if (members.size() < 2) continue;
        // longest run of identical leading blocks that is full in every member
        int64_t common = INT64_MAX;
        for (int i : members) common = std::min<int64_t>(common, seqs[i]->len / kBlockTokens);
        const Sequence &s0 = *seqs[members[0]];
        int64_t k = 0;
        while (k < common) {
            bool same = true;
            for (int i : members) same = same && seqs[i]->blocks[k] == s0.blocks[k];
            if (!same) break;
            ++k;
        }
        if (k == 0) continue;
        for (int i : members) {
            prefix_blocks_out[i] = static_cast<int32_t>(k);
            group_seqs_out[pos++] = i;
        }
        group_offsets_out[++groups] = pos;
    }
    *num_groups_out = groups;
    return PKV_OK;
}

extern "C" {

pkv_status pkv_alloc_refcount(const pkv_alloc *a, int64_t block, int32_t *out) {
    if (!a || !out || block < 0 || block >= a->num_blocks) return PKV_ERR_INVALID_ARG;
    *out = a->refcount[static_cast<size_t>(block)];
    return PKV_OK;
}

pkv_status pkv_alloc_seq_len(const pkv_alloc *a, int64_t seq_id, int64_t *len_out) {
    if (!a || !len_out) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
    *len_out = it->second.len;
    return PKV_OK;
}

pkv_status pkv_alloc_slot_of(const pkv_alloc *a, int64_t seq_id, int64_t pos, int64_t *slot_out) {
    if (!a || !slot_out) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || it->second.swapped || pos < 0 || pos >= it->second.len)
        return PKV_ERR_INVALID_ARG;
    *slot_out = static_cast<int64_t>(it->second.blocks[pos / kBlockTokens]) * kBlockTokens +
                pos % kBlockTokens;
    return PKV_OK;
}

}  // extern "C"
