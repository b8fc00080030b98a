// Host-side KV block pool (see include/pa_pool.h for the contract and the
// passages of "PagedAttention: fragmentation, blocks, block tables" and
// "Memory management" it follows).
//
// Data layout: reference counts in one int32 array indexed by block id; the
// free queue is a ring buffer of block ids with O(1) pop at the head and
// O(1) push at the head (frees are prepended, LIFO); sequences live in a hash
// map from id to {block list, token count, tail-owned flag}.

#include "pa_pool.h"

#include <algorithm>
#include <cstring>
#include <new>
#include <unordered_map>
#include <utility>
#include <vector>

namespace {

struct Seq {
    std::vector<int32_t> blocks;
    int64_t len = 0;
    bool tail_owned = true;  // false while the tail block is inherited from a fork
    uint64_t batch = 0;      // stamp of the last batch call that listed the sequence
};

// Ring buffer holding at most `cap` block ids; head() is the next to allocate.
class FreeRing {
  public:
    explicit FreeRing(int64_t cap) : buf_(static_cast<size_t>(cap)), cap_(cap) {}
    int64_t size() const { return size_; }
    int32_t pop_front() {
        int32_t b = buf_[static_cast<size_t>(head_)];
        head_ = (head_ + 1) % cap_;
        --size_;
        return b;
    }
    void push_front(int32_t b) {
        head_ = (head_ - 1 + cap_) % cap_;
        buf_[static_cast<size_t>(head_)] = b;
        ++size_;
    }
    void push_back(int32_t b) {
        buf_[static_cast<size_t>((head_ + size_) % cap_)] = b;
        ++size_;
    }
    int32_t at(int64_t i) const { return buf_[static_cast<size_t>((head_ + i) % cap_)]; }

  private:
    std::vector<int32_t> buf_;
    int64_t cap_;
    int64_t head_ = 0;
    int64_t size_ = 0;
};

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

struct pa_pool {
    int64_t num_blocks;
    int32_t block_size;
    int32_t rule;
    std::vector<int32_t> ref;  // owner references: tables naming the block
    std::vector<int32_t> pin;  // queued copies naming the block
    FreeRing free_q;
    std::unordered_map<int64_t, Seq> seqs;
    std::vector<std::pair<int32_t, int32_t>> pending;
    // Scratch of the batch calls, kept to avoid allocating per call: the
    // listed sequences in order, and per block the owner references earlier
    // appends of the batch move off it (reset before each call returns).
    uint64_t batch_epoch = 0;
    std::vector<Seq *> batch;
    std::vector<int32_t> moved;
    std::vector<int32_t> moved_touched;

    pa_pool(int64_t nb, int32_t bs, int32_t r)
        : num_blocks(nb), block_size(bs), rule(r), ref(static_cast<size_t>(nb), 0),
          pin(static_cast<size_t>(nb), 0), free_q(nb), moved(static_cast<size_t>(nb), 0) {}

    // Pop n blocks from the head of the free queue; each gets refcount 1.
    void take(int64_t n, std::vector<int32_t> &out) {
        for (int64_t i = 0; i < n; ++i) {
            int32_t b = free_q.pop_front();
            ref[static_cast<size_t>(b)] = 1;
            out.push_back(b);
        }
    }

    // Drop one reference (owner or pin, per `counts`) of each block in the
    // given order; blocks left with neither owners nor pins are pushed back at
    // the head of the free queue together, keeping that order.
    void release_refs(const int32_t *ordered, size_t n, std::vector<int32_t> &counts) {
        std::vector<int32_t> run;
        for (size_t i = 0; i < n; ++i) {
            const size_t b = static_cast<size_t>(ordered[i]);
            --counts[b];
            if (ref[b] == 0 && pin[b] == 0)
                run.push_back(ordered[i]);
        }
        for (size_t i = run.size(); i-- > 0;)
            free_q.push_front(run[i]);
    }
};

namespace {

// What appending n tokens to s takes: new blocks, and whether the partial
// tail is copied first.  Shared rule: the tail is copied while another table
// still names it; `moved_off_tail` counts owner references that earlier
// appends of the same batch will have moved off it.  Inherited rule: while
// the sequence has not written its forked tail.
struct AppendPlan {
    int64_t needed;
    bool cow;
};

AppendPlan plan_append(const pa_pool &pool, const Seq &s, int64_t n_tokens, int32_t moved_off_tail) {
    const int64_t B = pool.block_size;
    AppendPlan a;
    a.needed = cdiv(s.len + n_tokens, B) - static_cast<int64_t>(s.blocks.size());
    const bool partial = !s.blocks.empty() && s.len % B != 0 && n_tokens > 0;
    if (pool.rule == PA_COW_SHARED)
        a.cow = partial && pool.ref[static_cast<size_t>(s.blocks.back())] - moved_off_tail > 1;
    else
        a.cow = partial && !s.tail_owned;
    return a;
}

bool too_long(const pa_pool &pool, const Seq &s, int64_t n_tokens) {
    // more than the whole pool holds (this also keeps len + n_tokens in range)
    return n_tokens > pool.num_blocks * pool.block_size - s.len;
}

// Carry out an append whose blocks the caller has checked are free.
void apply_append(pa_pool &pool, Seq &s, int64_t n_tokens, const AppendPlan &a) {
    if (a.cow) {
        const int32_t src = s.blocks.back();
        const int32_t dst = pool.free_q.pop_front();
        pool.ref[static_cast<size_t>(dst)] = 1;
        // The sequence stops owning src; both ends stay pinned until the
        // copy is handed to the device.
        pool.ref[static_cast<size_t>(src)] -= 1;
        pool.pin[static_cast<size_t>(src)] += 1;
        pool.pin[static_cast<size_t>(dst)] += 1;
        s.blocks.back() = dst;
        pool.pending.emplace_back(src, dst);
        s.tail_owned = true;
    }
    if (a.needed > 0) {
        pool.take(a.needed, s.blocks);
        s.tail_owned = true;
    }
    s.len += n_tokens;
}

// Dry run of appending n_tokens to each listed sequence in call order, with
// the copy-on-write decisions of the earlier ones applied (a copy takes a
// sequence off its shared tail, which a later sharer may then own alone).
// Leaves the sequences in pool.batch; adds up the free blocks and the copies
// the appends need.  Changes no visible state.
int plan_batch(pa_pool &pool, const int64_t *seq_ids, int32_t num_seqs, int64_t n_tokens, int64_t &blocks,
               int64_t &copies) {
    const uint64_t stamp = ++pool.batch_epoch;
    pool.batch.clear();
    pool.moved_touched.clear();
    blocks = copies = 0;
    int rc = PA_POOL_OK;
    for (int32_t i = 0; i < num_seqs; ++i) {
        auto it = pool.seqs.find(seq_ids[i]);
        if (it == pool.seqs.end()) {
            rc = PA_POOL_ENOSEQ;
            break;
        }
        Seq &s = it->second;
        if (s.batch == stamp) {
            rc = PA_POOL_EINVAL;  // a sequence listed twice
            break;
        }
        s.batch = stamp;
        if (too_long(pool, s, n_tokens)) {
            rc = PA_POOL_ENOSPACE;
            break;
        }
        const int32_t tail = s.blocks.empty() ? -1 : s.blocks.back();
        const AppendPlan a = plan_append(pool, s, n_tokens, tail >= 0 ? pool.moved[static_cast<size_t>(tail)] : 0);
        if (a.cow && pool.rule == PA_COW_SHARED) {
            if (pool.moved[static_cast<size_t>(tail)]++ == 0)
                pool.moved_touched.push_back(tail);
        }
        blocks += a.needed + (a.cow ? 1 : 0);
        copies += a.cow ? 1 : 0;
        pool.batch.push_back(&s);
    }
    for (int32_t b : pool.moved_touched)
        pool.moved[static_cast<size_t>(b)] = 0;
    return rc;
}

// Append to every sequence of pool.batch (after a successful plan_batch
// whose blocks are free): each decision is taken again on the live state,
// which by then matches the dry run's.
void apply_batch(pa_pool &pool, int64_t n_tokens) {
    for (Seq *s : pool.batch)
        apply_append(pool, *s, n_tokens, plan_append(pool, *s, n_tokens, 0));
}

// Move the queued pairs to pairs_out (capacity checked by the caller) and
// drop the pins their endpoints held.
int64_t take_copies(pa_pool &pool, int64_t *pairs_out) {
    const int64_t n = static_cast<int64_t>(pool.pending.size());
    std::vector<std::pair<int32_t, int32_t>> taken;
    taken.swap(pool.pending);
    for (int64_t i = 0; i < n; ++i) {
        pairs_out[2 * i] = taken[static_cast<size_t>(i)].first;
        pairs_out[2 * i + 1] = taken[static_cast<size_t>(i)].second;
        const int32_t ends[2] = {taken[static_cast<size_t>(i)].first, taken[static_cast<size_t>(i)].second};
        pool.release_refs(ends, 2, pool.pin);
    }
    taken.clear();
    taken.swap(pool.pending);  // keep the capacity for the next step
    return n;
}

// Rewrite the entries of a table row that can have changed since `synced`
// of them were written: the old tail (a copy-on-write may have redirected
// it) and every entry after it.
void update_row(const Seq &s, int32_t *row, int32_t &synced) {
    const int32_t n = static_cast<int32_t>(s.blocks.size());
    const int32_t from = synced > 0 ? synced - 1 : 0;
    std::copy(s.blocks.begin() + from, s.blocks.end(), row + from);
    synced = n;
}

}  // namespace

extern "C" {

pa_pool_t *pa_pool_create(int64_t num_blocks, int32_t block_size, const int32_t *free_order,
                          int32_t cow_rule) {
    if (num_blocks <= 0 || num_blocks > INT32_MAX || block_size <= 0 ||
        (cow_rule != PA_COW_SHARED && cow_rule != PA_COW_INHERITED))
        return nullptr;
    pa_pool *p = new (std::nothrow) pa_pool(num_blocks, block_size, cow_rule);
    if (!p)
        return nullptr;
    if (free_order) {
        std::vector<char> seen(static_cast<size_t>(num_blocks), 0);
        for (int64_t i = 0; i < num_blocks; ++i) {
            int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[static_cast<size_t>(b)]) {
                delete p;
                return nullptr;
            }
            seen[static_cast<size_t>(b)] = 1;
            p->free_q.push_back(b);
        }
    } else {
        for (int64_t i = 0; i < num_blocks; ++i)
            p->free_q.push_back(static_cast<int32_t>(i));
    }
    return p;
}

void pa_pool_destroy(pa_pool_t *pool) { delete pool; }

int pa_pool_seq_create(pa_pool_t *pool, int64_t seq_id) {
    if (!pool)
        return PA_POOL_EINVAL;
    if (pool->seqs.count(seq_id))
        return PA_POOL_EEXIST;
    pool->seqs.emplace(seq_id, Seq{});
    return PA_POOL_OK;
}

int pa_pool_append(pa_pool_t *pool, int64_t seq_id, int64_t n_tokens) {
    if (!pool || n_tokens < 0)
        return PA_POOL_EINVAL;
    auto it = pool->seqs.find(seq_id);
    if (it == pool->seqs.end())
        return PA_POOL_ENOSEQ;
    Seq &s = it->second;
    if (too_long(*pool, s, n_tokens))
        return PA_POOL_ENOSPACE;
    const AppendPlan a = plan_append(*pool, s, n_tokens, 0);
    if (a.needed + (a.cow ? 1 : 0) > pool->free_q.size())
        return PA_POOL_ENOSPACE;
    apply_append(*pool, s, n_tokens, a);
    return PA_POOL_OK;
}

int pa_pool_append_batch(pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs, int64_t n_tokens) {
    if (!pool || n_tokens < 0 || num_seqs < 0 || (num_seqs > 0 && !seq_ids))
        return PA_POOL_EINVAL;
    int64_t blocks = 0, copies = 0;
    const int rc = plan_batch(*pool, seq_ids, num_seqs, n_tokens, blocks, copies);
    if (rc != PA_POOL_OK)
        return rc;
    if (blocks > pool->free_q.size())
        return PA_POOL_ENOSPACE;
    apply_batch(*pool, n_tokens);
    return PA_POOL_OK;
}

int pa_pool_step(pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs, int64_t n_tokens, int64_t *pairs_out,
                 int64_t pairs_capacity, int64_t *num_pairs, int64_t *slots_out, int32_t width, int32_t *table,
                 int32_t *synced, int32_t *lens_out) {
    if (!pool || n_tokens < 0 || num_seqs < 0 || width < 0 || pairs_capacity < 0 || !num_pairs ||
        (num_seqs > 0 && (!seq_ids || !table || !synced || !lens_out || (n_tokens > 0 && !slots_out))))
        return PA_POOL_EINVAL;
    int64_t blocks = 0, copies = 0;
    int rc = plan_batch(*pool, seq_ids, num_seqs, n_tokens, blocks, copies);
    if (rc != PA_POOL_OK)
        return rc;
    if (blocks > pool->free_q.size())
        return PA_POOL_ENOSPACE;
    const int64_t npairs = static_cast<int64_t>(pool->pending.size()) + copies;
    if (npairs > pairs_capacity || (npairs > 0 && !pairs_out))
        return PA_POOL_ERANGE;
    const int64_t B = pool->block_size;
    for (int32_t r = 0; r < num_seqs; ++r) {
        const Seq &s = *pool->batch[static_cast<size_t>(r)];
        if (cdiv(s.len + n_tokens, B) > width || synced[r] < 0 || synced[r] > width || s.len + n_tokens > INT32_MAX)
            return PA_POOL_ERANGE;
        if (synced[r] > static_cast<int64_t>(s.blocks.size()))
            return PA_POOL_EINVAL;  // the row was not reset for this sequence
    }
    // Every check is done: nothing below can fail.
    apply_batch(*pool, n_tokens);
    *num_pairs = take_copies(*pool, pairs_out);
    for (int32_t r = 0; r < num_seqs; ++r) {
        const Seq &s = *pool->batch[static_cast<size_t>(r)];
        int64_t *out = slots_out + static_cast<int64_t>(r) * n_tokens;
        for (int64_t i = 0; i < n_tokens; ++i) {
            const int64_t pos = s.len - n_tokens + i;
            out[i] = static_cast<int64_t>(s.blocks[static_cast<size_t>(pos / B)]) * B + pos % B;
        }
        update_row(s, table + static_cast<int64_t>(r) * width, synced[r]);
        lens_out[r] = static_cast<int32_t>(s.len);
    }
    return PA_POOL_OK;
}

int pa_pool_fork(pa_pool_t *pool, int64_t src, int64_t dst) {
    if (!pool)
        return PA_POOL_EINVAL;
    auto it = pool->seqs.find(src);
    if (it == pool->seqs.end())
        return PA_POOL_ENOSEQ;
    if (pool->seqs.count(dst))
        return PA_POOL_EEXIST;
    Seq child;
    child.blocks = it->second.blocks;
    child.len = it->second.len;
    child.tail_owned = child.blocks.empty();
    for (int32_t b : child.blocks)
        pool->ref[static_cast<size_t>(b)] += 1;
    pool->seqs.emplace(dst, std::move(child));
    return PA_POOL_OK;
}

int pa_pool_release(pa_pool_t *pool, int64_t seq_id) {
    if (!pool)
        return PA_POOL_EINVAL;
    auto it = pool->seqs.find(seq_id);
    if (it == pool->seqs.end())
        return PA_POOL_ENOSEQ;
    std::vector<int32_t> rev(it->second.blocks.rbegin(), it->second.blocks.rend());
    pool->seqs.erase(it);
    pool->release_refs(rev.data(), rev.size(), pool->ref);
    return PA_POOL_OK;
}

int64_t pa_pool_num_pending_copies(const pa_pool_t *pool) {
    return pool ? static_cast<int64_t>(pool->pending.size()) : static_cast<int64_t>(PA_POOL_EINVAL);
}

int64_t pa_pool_take_copies(pa_pool_t *pool, int64_t *pairs_out, int64_t capacity) {
    if (!pool)
        return PA_POOL_EINVAL;
    const int64_t n = static_cast<int64_t>(pool->pending.size());
    if (n > capacity || (n > 0 && !pairs_out))
        return PA_POOL_ERANGE;
    return take_copies(*pool, pairs_out);
}

int64_t pa_pool_num_blocks(const pa_pool_t *pool) {
    return pool ? pool->num_blocks : static_cast<int64_t>(PA_POOL_EINVAL);
}
int32_t pa_pool_block_size(const pa_pool_t *pool) {
    return pool ? pool->block_size : static_cast<int32_t>(PA_POOL_EINVAL);
}
int64_t pa_pool_num_free(const pa_pool_t *pool) {
    return pool ? pool->free_q.size() : static_cast<int64_t>(PA_POOL_EINVAL);
}

int64_t pa_pool_seq_len(const pa_pool_t *pool, int64_t seq_id) {
    if (!pool)
        return PA_POOL_EINVAL;
    auto it = pool->seqs.find(seq_id);
    return it == pool->seqs.end() ? static_cast<int64_t>(PA_POOL_ENOSEQ) : it->second.len;
}

int64_t pa_pool_seq_num_blocks(const pa_pool_t *pool, int64_t seq_id) {
    if (!pool)
        return PA_POOL_EINVAL;
    auto it = pool->seqs.find(seq_id);
    return it == pool->seqs.end() ? static_cast<int64_t>(PA_POOL_ENOSEQ)
                                  : static_cast<int64_t>(it->second.blocks.size());
}

int32_t pa_pool_refcount(const pa_pool_t *pool, int64_t block) {
    if (!pool || block < 0 || block >= pool->num_blocks)
        return PA_POOL_EINVAL;
    return pool->ref[static_cast<size_t>(block)];
}

int32_t pa_pool_pins(const pa_pool_t *pool, int64_t block) {
    if (!pool || block < 0 || block >= pool->num_blocks)
        return PA_POOL_EINVAL;
    return pool->pin[static_cast<size_t>(block)];
}

int64_t pa_pool_free_list(const pa_pool_t *pool, int32_t *out, int64_t capacity) {
    if (!pool)
        return PA_POOL_EINVAL;
    const int64_t n = pool->free_q.size();
    if (n > capacity || (n > 0 && !out))
        return PA_POOL_ERANGE;
    for (int64_t i = 0; i < n; ++i)
        out[i] = pool->free_q.at(i);
    return n;
}

int pa_pool_block_table(const pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs,
                        int32_t width, int32_t pad, int32_t *out) {
    if (!pool || num_seqs < 0 || width < 0 || (num_seqs > 0 && (!seq_ids || !out)))
        return PA_POOL_EINVAL;
    for (int32_t r = 0; r < num_seqs; ++r) {
        auto it = pool->seqs.find(seq_ids[r]);
        if (it == pool->seqs.end())
            return PA_POOL_ENOSEQ;
        if (static_cast<int64_t>(it->second.blocks.size()) > width)
            return PA_POOL_ERANGE;
    }
    for (int32_t r = 0; r < num_seqs; ++r) {
        const std::vector<int32_t> &bl = pool->seqs.find(seq_ids[r])->second.blocks;
        int32_t *row = out + static_cast<int64_t>(r) * width;
        std::copy(bl.begin(), bl.end(), row);
        std::fill(row + bl.size(), row + width, pad);
    }
    return PA_POOL_OK;
}

int pa_pool_block_table_update(const pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs, int32_t width,
                               int32_t /* pad: rows past their count already hold it */, int32_t *out,
                               int32_t *synced) {
    if (!pool || num_seqs < 0 || width < 0 || (num_seqs > 0 && (!seq_ids || !out || !synced)))
        return PA_POOL_EINVAL;
    for (int32_t r = 0; r < num_seqs; ++r) {
        auto it = pool->seqs.find(seq_ids[r]);
        if (it == pool->seqs.end())
            return PA_POOL_ENOSEQ;
        const int64_t n = static_cast<int64_t>(it->second.blocks.size());
        if (n > width || synced[r] < 0 || synced[r] > width)
            return PA_POOL_ERANGE;
        if (synced[r] > n)  // a sequence never loses blocks: the row names another one now
            return PA_POOL_EINVAL;
    }
    for (int32_t r = 0; r < num_seqs; ++r)
        update_row(pool->seqs.find(seq_ids[r])->second, out + static_cast<int64_t>(r) * width, synced[r]);
    return PA_POOL_OK;
}

int pa_pool_seq_lens(const pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs, int32_t *out) {
    if (!pool || num_seqs < 0 || (num_seqs > 0 && (!seq_ids || !out)))
        return PA_POOL_EINVAL;
    for (int32_t r = 0; r < num_seqs; ++r) {
        auto it = pool->seqs.find(seq_ids[r]);
        if (it == pool->seqs.end())
            return PA_POOL_ENOSEQ;
        if (it->second.len > INT32_MAX)
            return PA_POOL_ERANGE;
        out[r] = static_cast<int32_t>(it->second.len);
    }
    return PA_POOL_OK;
}

int pa_pool_slots(const pa_pool_t *pool, int64_t seq_id, int64_t pos0, int64_t count, int64_t *out) {
    if (!pool || pos0 < 0 || count < 0 || (count > 0 && !out))
        return PA_POOL_EINVAL;
    auto it = pool->seqs.find(seq_id);
    if (it == pool->seqs.end())
        return PA_POOL_ENOSEQ;
    const Seq &s = it->second;
    if (pos0 + count > s.len)
        return PA_POOL_ERANGE;
    const int64_t B = pool->block_size;
    for (int64_t i = 0; i < count; ++i) {
        const int64_t p = pos0 + i;
        out[i] = static_cast<int64_t>(s.blocks[static_cast<size_t>(p / B)]) * B + p % B;
    }
    return PA_POOL_OK;
}

int pa_pool_step_slots(const pa_pool_t *pool, const int64_t *seq_ids, int32_t num_seqs,
                       int64_t tokens_per_seq, int64_t *out) {
    if (!pool || num_seqs < 0 || tokens_per_seq < 0 || (num_seqs > 0 && (!seq_ids || !out)))
        return PA_POOL_EINVAL;
    for (int32_t r = 0; r < num_seqs; ++r) {
        const int64_t len = pa_pool_seq_len(pool, seq_ids[r]);
        if (len < 0)
            return static_cast<int>(len);
        if (len < tokens_per_seq)
            return PA_POOL_ERANGE;
    }
    for (int32_t r = 0; r < num_seqs; ++r) {
        const int64_t len = pool->seqs.find(seq_ids[r])->second.len;
        pa_pool_slots(pool, seq_ids[r], len - tokens_per_seq, tokens_per_seq,
                      out + static_cast<int64_t>(r) * tokens_per_seq);
    }
    return PA_POOL_OK;
}

int pa_pool_check(const pa_pool_t *pool) {
    if (!pool)
        return PA_POOL_EINVAL;
    const size_t nb = static_cast<size_t>(pool->num_blocks);
    std::vector<int64_t> counted(nb, 0), pinned(nb, 0);
    std::vector<char> on_free(nb, 0);
    for (int64_t i = 0; i < pool->free_q.size(); ++i) {
        const int32_t b = pool->free_q.at(i);
        if (b < 0 || static_cast<size_t>(b) >= nb || on_free[static_cast<size_t>(b)])
            return PA_POOL_EINVARIANT;
        on_free[static_cast<size_t>(b)] = 1;
    }
    const int64_t B = pool->block_size;
    std::vector<int32_t> sorted;
    for (const auto &kv : pool->seqs) {
        const Seq &s = kv.second;
        if (static_cast<int64_t>(s.blocks.size()) != cdiv(s.len, B))
            return PA_POOL_EINVARIANT;
        sorted = s.blocks;
        std::sort(sorted.begin(), sorted.end());
        if (std::adjacent_find(sorted.begin(), sorted.end()) != sorted.end())
            return PA_POOL_EINVARIANT;
        for (int32_t b : s.blocks)
            counted[static_cast<size_t>(b)] += 1;
    }
    for (const auto &pr : pool->pending) {
        pinned[static_cast<size_t>(pr.first)] += 1;
        pinned[static_cast<size_t>(pr.second)] += 1;
    }
    for (size_t b = 0; b < nb; ++b) {
        if (counted[b] != pool->ref[b] || pinned[b] != pool->pin[b])
            return PA_POOL_EINVARIANT;
        if ((on_free[b] != 0) == (pool->ref[b] + pool->pin[b] > 0))
            return PA_POOL_EINVARIANT;
    }
    return PA_POOL_OK;
}

const char *pa_pool_status_str(int status) {
    switch (status) {
    case PA_POOL_OK: return "ok";
    case PA_POOL_EINVAL: return "invalid argument";
    case PA_POOL_ENOSPACE: return "not enough free blocks (pool unchanged)";
    case PA_POOL_ENOSEQ: return "unknown sequence id";
    case PA_POOL_EEXIST: return "sequence id already in use";
    case PA_POOL_EINVARIANT: return "allocator invariant broken";
    case PA_POOL_ERANGE: return "output too small or position out of range";
    default: return "unknown status";
    }
}

}  // extern "C"
