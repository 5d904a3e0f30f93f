// Host block manager of the paged KV cache (include/pa_block_manager.h).
//
// A pool of reference-counted blocks, a LIFO free list and, per sequence, its page
// table (physical block ids in token order) and length.  Allocation is on demand;
// a sequence that appends into a shared, partially filled last block gets a private
// copy first (copy-on-write), reported as a (src, dst) pair for pa_copy_blocks.
// Under a sliding window of W tokens, a block that lies wholly before the last W
// positions of its sequence is given back and its table entry becomes -1.
//
// Failure atomicity: every entry point either does all of its work or changes nothing.
// Those that allocate host memory do every allocation (or reserve the capacity they
// will fill) before the first change, and a failed allocation becomes
// PA_ERR_HOST_ALLOC at the C boundary instead of an exception.  The free lists never
// grow past the capacity reserved when their pool was made, so giving blocks back
// cannot fail.
#include <cstdint>
#include <memory>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa_block_manager.h"

struct pa_block_manager {
    int num_blocks = 0;
    int block_size = 0;
    std::vector<int> refcount;   // per physical block, 0 = free
    std::vector<int> free_list;  // LIFO of free block ids
    struct Seq {
        std::vector<int> blocks;  // GPU block ids, or host block ids when on_cpu; -1 = released
        int len = 0;
        int first_live = 0;  // blocks[0 .. first_live) were released (sliding window)
        unsigned stamp = 0;  // last append batch that listed this sequence
        bool on_cpu = false;
    };
    // host pool (preemption)
    int num_cpu_blocks = 0;
    std::vector<int> cpu_refcount;
    std::vector<int> cpu_free_list;
    std::unordered_map<int64_t, Seq> seqs;
    // scratch of pa_bm_append_slots: references to a block given up earlier in the
    // current batch, valid where released_stamp[block] == batch
    std::vector<int> released;
    std::vector<unsigned> released_stamp;
    std::vector<Seq *> batch_seqs;
    unsigned batch = 0;
    int window = 0;  // sliding window in tokens, 0 = whole contexts

    // Blocks of a context of n tokens that lie wholly before its window.
    int blocks_before_window(int n) const {
        return (window > 0 && n > window) ? (n - window) / block_size : 0;
    }
    void release_before_window(Seq &s) {
        const int upto = blocks_before_window(s.len);
        for (int j = s.first_live; j < upto; ++j) {
            drop(s.blocks[j]);
            s.blocks[j] = -1;
        }
        if (upto > s.first_live) s.first_live = upto;
    }

    int take() {  // caller checked that the free list is not empty
        const int b = free_list.back();
        free_list.pop_back();
        refcount[b] = 1;
        return b;
    }
    void drop(int b) {
        if (--refcount[b] == 0) free_list.push_back(b);
    }
};

namespace {

// Runs an entry point's body; an exception (a failed host allocation) becomes
// PA_ERR_HOST_ALLOC.  The bodies allocate before they change anything.
template <typename Body>
pa_status no_throw(Body &&body) {
    try {
        return body();
    } catch (...) {
        return PA_ERR_HOST_ALLOC;
    }
}

// Moves the listed sequences between the pools: `from` (refcounts, free list) -> `to`.
pa_status move_group(pa_block_manager *bm, const int64_t *seq_ids, int n, int64_t *pairs,
                     int max_pairs, int *num_pairs, bool out) {
    if (!bm || n < 0 || (n > 0 && !seq_ids) || !num_pairs || max_pairs < 0 ||
        (max_pairs > 0 && !pairs))
        return PA_ERR_INVALID_ARG;
    if (out && bm->num_cpu_blocks == 0) return PA_ERR_INVALID_ARG;
    std::vector<int> &from_ref = out ? bm->refcount : bm->cpu_refcount;
    std::vector<int> &to_ref = out ? bm->cpu_refcount : bm->refcount;
    std::vector<int> &from_free = out ? bm->free_list : bm->cpu_free_list;
    std::vector<int> &to_free = out ? bm->cpu_free_list : bm->free_list;
    std::vector<pa_block_manager::Seq *> group;
    std::unordered_map<int, int> uses;  // block -> references held by the group
    std::vector<int> order;             // distinct blocks, first-use order
    for (int i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end() || it->second.on_cpu != !out) return PA_ERR_INVALID_ARG;
        for (pa_block_manager::Seq *g : group)
            if (g == &it->second) return PA_ERR_INVALID_ARG;  // listed twice
        group.push_back(&it->second);
        for (int b : it->second.blocks)
            if (b >= 0 && uses[b]++ == 0) order.push_back(b);
    }
    for (int b : order)
        if (uses[b] != from_ref[b]) return PA_ERR_INVALID_ARG;  // shared outside the group
    if ((int)order.size() > (int)to_free.size()) return PA_ERR_NO_FREE_BLOCK;
    if ((int)order.size() > max_pairs) return PA_ERR_INVALID_ARG;
    // the destination of every block, decided (and allocated) before anything moves
    std::unordered_map<int, int> moved;
    moved.reserve(order.size());
    for (size_t i = 0; i < order.size(); ++i)
        moved.emplace(order[i], to_free[to_free.size() - 1 - i]);
    for (size_t i = 0; i < order.size(); ++i) {
        const int b = order[i];
        const int nb = to_free.back();
        to_free.pop_back();
        to_ref[nb] = from_ref[b];
        from_ref[b] = 0;
        from_free.push_back(b);  // within the capacity reserved for that pool
        pairs[2 * i] = b;
        pairs[2 * i + 1] = nb;
    }
    for (pa_block_manager::Seq *g : group) {
        for (int &b : g->blocks)
            if (b >= 0) b = moved.find(b)->second;
        g->on_cpu = out;
    }
    *num_pairs = (int)order.size();
    return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_bm_set_cpu_pool(pa_block_manager *bm, int num_cpu_blocks) {
    if (!bm || num_cpu_blocks <= 0 || bm->num_cpu_blocks != 0) return PA_ERR_INVALID_ARG;
    return no_throw([&] {
        std::vector<int> ref(num_cpu_blocks, 0), free_list;
        free_list.reserve(num_cpu_blocks);
        for (int b = num_cpu_blocks - 1; b >= 0; --b) free_list.push_back(b);
        bm->cpu_refcount.swap(ref);
        bm->cpu_free_list.swap(free_list);
        bm->num_cpu_blocks = num_cpu_blocks;
        return PA_OK;
    });
}

int pa_bm_num_free_cpu_blocks(const pa_block_manager *bm) {
    return bm ? (int)bm->cpu_free_list.size() : 0;
}

int pa_bm_is_swapped(const pa_block_manager *bm, int64_t seq_id) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : (it->second.on_cpu ? 1 : 0);
}

pa_status pa_bm_swap_out(pa_block_manager *bm, const int64_t *seq_ids, int n, int64_t *pairs,
                         int max_pairs, int *num_pairs) {
    return no_throw([&] { return move_group(bm, seq_ids, n, pairs, max_pairs, num_pairs, true); });
}

pa_status pa_bm_swap_in(pa_block_manager *bm, const int64_t *seq_ids, int n, int64_t *pairs,
                        int max_pairs, int *num_pairs) {
    return no_throw(
        [&] { return move_group(bm, seq_ids, n, pairs, max_pairs, num_pairs, false); });
}

pa_status pa_bm_set_sliding_window(pa_block_manager *bm, int window) {
    if (!bm || window < 0 || !bm->seqs.empty()) return PA_ERR_INVALID_ARG;
    bm->window = window;
    return PA_OK;
}

pa_block_manager *pa_bm_create(int num_blocks, int block_size) {
    if (num_blocks <= 0 || block_size <= 0) return nullptr;
    try {
        std::unique_ptr<pa_block_manager> bm(new pa_block_manager());
        bm->num_blocks = num_blocks;
        bm->block_size = block_size;
        bm->refcount.assign(num_blocks, 0);
        bm->released.assign(num_blocks, 0);
        bm->released_stamp.assign(num_blocks, 0);
        bm->free_list.reserve(num_blocks);
        for (int b = num_blocks - 1; b >= 0; --b) bm->free_list.push_back(b);  // hands out 0, 1, ...
        return bm.release();
    } catch (...) {
        return nullptr;  // out of host memory
    }
}

void pa_bm_destroy(pa_block_manager *bm) { delete bm; }

int pa_bm_blocks_needed(int num_tokens, int block_size) {
    if (num_tokens < 0 || block_size <= 0) return -1;
    return (int)(((long long)num_tokens + block_size - 1) / block_size);
}

int pa_bm_num_free_blocks(const pa_block_manager *bm) {
    return bm ? (int)bm->free_list.size() : 0;
}

double pa_bm_usage_ratio(const pa_block_manager *bm) {
    if (!bm || bm->num_blocks == 0) return 0.0;
    return (double)(bm->num_blocks - (int)bm->free_list.size()) / bm->num_blocks;
}

int pa_bm_can_allocate(const pa_block_manager *bm, int num_tokens) {
    if (!bm) return 0;
    const int need = pa_bm_blocks_needed(num_tokens, bm->block_size);
    return need >= 0 && need <= (int)bm->free_list.size();
}

pa_status pa_bm_allocate(pa_block_manager *bm, int64_t seq_id, int num_tokens) {
    if (!bm || num_tokens < 0 || bm->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
    // every token of a prompt is written and attended (prefill), so a new sequence
    // takes all its blocks; those before the window go back at its next append
    const int need = pa_bm_blocks_needed(num_tokens, bm->block_size);
    if (need > (int)bm->free_list.size()) return PA_ERR_NO_FREE_BLOCK;
    return no_throw([&] {
        pa_block_manager::Seq s;
        s.blocks.reserve(need);
        pa_block_manager::Seq &t = bm->seqs.emplace(seq_id, std::move(s)).first->second;
        for (int i = 0; i < need; ++i) t.blocks.push_back(bm->take());  // within capacity
        t.len = num_tokens;
        return PA_OK;
    });
}

pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent_id, int64_t child_id) {
    if (!bm || parent_id == child_id) return PA_ERR_INVALID_ARG;
    auto it = bm->seqs.find(parent_id);
    if (it == bm->seqs.end() || it->second.on_cpu || bm->seqs.count(child_id))
        return PA_ERR_INVALID_ARG;
    return no_throw([&] {
        // the copy and the insertion allocate; the reference counts change after them
        pa_block_manager::Seq &child = bm->seqs.emplace(child_id, it->second).first->second;
        child.stamp = 0;
        for (int b : child.blocks)
            if (b >= 0) ++bm->refcount[b];
        return PA_OK;
    });
}

pa_status pa_bm_free(pa_block_manager *bm, int64_t seq_id) {
    if (!bm) return PA_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
    // return blocks back to front, so the next allocation reuses them in order
    for (auto b = it->second.blocks.rbegin(); b != it->second.blocks.rend(); ++b) {
        if (*b < 0) continue;  // released (sliding window)
        if (it->second.on_cpu) {
            if (--bm->cpu_refcount[*b] == 0) bm->cpu_free_list.push_back(*b);
        } else {
            bm->drop(*b);
        }
    }
    bm->seqs.erase(it);
    return PA_OK;
}

namespace {

// pa_bm_append_slots, reporting each private copy as a pair (copy_pairs) or per sequence
// (cow: source block, logical index of the copied block, rows filled before the token).
pa_status append_slots(pa_block_manager *bm, const int64_t *seq_ids, int n,
                       int64_t *slot_mapping, int64_t *copy_pairs, int max_pairs,
                       int *num_pairs, int32_t *cow) {
    const int bs = bm->block_size;
    // pass 1: validate and count the fresh blocks the batch needs (without changing
    // anything), following the reference counts as earlier entries of the batch
    // would change them
    const unsigned stamp = ++bm->batch;
    if (no_throw([&] {
            bm->batch_seqs.resize(n);
            return PA_OK;
        }) != PA_OK)
        return PA_ERR_HOST_ALLOC;
    int fresh = 0, pairs = 0;
    for (int i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end() || it->second.stamp == stamp || it->second.on_cpu) {
            for (int j = 0; j < i; ++j) bm->batch_seqs[j]->stamp = 0;
            return PA_ERR_INVALID_ARG;
        }
        pa_block_manager::Seq &s = it->second;
        s.stamp = stamp;
        bm->batch_seqs[i] = &s;
        if (s.len % bs == 0) {
            ++fresh;
            // room for the block pass 2 appends, so that pass 2 cannot fail half-way
            std::vector<int> &b = s.blocks;
            if (b.size() == b.capacity() &&
                no_throw([&] {
                    b.reserve(b.empty() ? 4 : 2 * b.size());
                    return PA_OK;
                }) != PA_OK) {
                for (int j = 0; j <= i; ++j) bm->batch_seqs[j]->stamp = 0;
                return PA_ERR_HOST_ALLOC;
            }
        } else {
            const int last = s.blocks.back();
            int &rel = bm->released[last];
            if (bm->released_stamp[last] != stamp) {
                bm->released_stamp[last] = stamp;
                rel = 0;
            }
            if (bm->refcount[last] - rel > 1) {
                ++fresh;
                ++pairs;
                ++rel;
            }
        }
    }
    if (fresh > (int)bm->free_list.size() || pairs > max_pairs) {
        for (int i = 0; i < n; ++i) bm->batch_seqs[i]->stamp = 0;
        return fresh > (int)bm->free_list.size() ? PA_ERR_NO_FREE_BLOCK : PA_ERR_INVALID_ARG;
    }
    // pass 2: apply
    int np = 0;
    for (int i = 0; i < n; ++i) {
        pa_block_manager::Seq &s = *bm->batch_seqs[i];
        const int off = s.len % bs;
        int blk;
        if (off == 0) {
            blk = bm->take();
            s.blocks.push_back(blk);  // within the capacity reserved in pass 1
        } else {
            blk = s.blocks.back();
            if (bm->refcount[blk] > 1) {
                const int copy = bm->take();
                if (copy_pairs) {
                    copy_pairs[2 * np] = blk;
                    copy_pairs[2 * np + 1] = copy;
                }
                if (cow) {
                    cow[3 * i] = blk;
                    cow[3 * i + 1] = (int32_t)s.blocks.size() - 1;
                    cow[3 * i + 2] = off;
                }
                ++np;
                bm->drop(blk);
                s.blocks.back() = copy;
                blk = copy;
            }
        }
        slot_mapping[i] = (int64_t)blk * bs + off;
        ++s.len;
    }
    // pass 3: blocks that fell out of the window of their sequence go back to the pool
    if (bm->window > 0)
        for (int i = 0; i < n; ++i) bm->release_before_window(*bm->batch_seqs[i]);
    *num_pairs = np;
    return PA_OK;
}

}  // namespace

pa_status pa_bm_append_slots(pa_block_manager *bm, const int64_t *seq_ids, int n,
                             int64_t *slot_mapping, int64_t *copy_pairs, int max_pairs,
                             int *num_pairs) {
    if (!bm || n < 0 || (n > 0 && (!seq_ids || !slot_mapping)) || !num_pairs || max_pairs < 0 ||
        (max_pairs > 0 && !copy_pairs))
        return PA_ERR_INVALID_ARG;
    return append_slots(bm, seq_ids, n, slot_mapping, copy_pairs, max_pairs, num_pairs,
                        nullptr);
}

pa_status pa_bm_append_slots_cow(pa_block_manager *bm, const int64_t *seq_ids, int n,
                                 int64_t *slot_mapping, int32_t *cow, int *num_copies) {
    if (!bm || n < 0 || (n > 0 && (!seq_ids || !slot_mapping || !cow)) || !num_copies)
        return PA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {  // no copy unless pass 2 records one
        cow[3 * i] = -1;
        cow[3 * i + 1] = 0;
        cow[3 * i + 2] = 0;
    }
    // at most one copy per listed sequence, so the pair bound never binds
    return append_slots(bm, seq_ids, n, slot_mapping, nullptr, n, num_copies, cow);
}

int64_t pa_bm_slot(const pa_block_manager *bm, int64_t seq_id, int pos) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || it->second.on_cpu || pos < 0 || pos >= it->second.len) return -1;
    const int blk = it->second.blocks[pos / bm->block_size];
    if (blk < 0) return -1;  // released (sliding window)
    return (int64_t)blk * bm->block_size + pos % bm->block_size;
}

int pa_bm_seq_len(const pa_block_manager *bm, int64_t seq_id) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : it->second.len;
}

int pa_bm_block_refcount(const pa_block_manager *bm, int block) {
    if (!bm || block < 0 || block >= bm->num_blocks) return -1;
    return bm->refcount[block];
}

pa_status pa_bm_block_tables(const pa_block_manager *bm, const int64_t *seq_ids, int n,
                             int32_t *block_tables, int width, int32_t *context_lens) {
    if (!bm || n < 0 || width <= 0 || (n > 0 && (!seq_ids || !block_tables || !context_lens)))
        return PA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end() || it->second.on_cpu ||
            (int)it->second.blocks.size() > width)
            return PA_ERR_INVALID_ARG;
        const std::vector<int> &b = it->second.blocks;
        for (int j = 0; j < width; ++j)
            block_tables[(size_t)i * width + j] = j < (int)b.size() ? b[j] : -1;
        context_lens[i] = it->second.len;
    }
    return PA_OK;
}

}  // extern "C"
