// Host block manager for the paged KV cache.
//
// Rules from "Memory Optimization in LLM Serving with PagedAttention":
//   section "How PagedAttention Works" -- the pool is cut into equal blocks; a sequence's
//   logical blocks map to physical blocks through its block table; blocks are taken only
//   when generation needs them, so only a sequence's last block can be partly empty;
//   section "Advanced Capabilities: Memory Sharing with Copy-on-Write" -- forked samples map
//   the same physical blocks; before a sequence appends into a block whose reference count
//   is above one it takes a fresh block, has the content copied there, repoints its own
//   table entry, and only then writes.
// The free list is first-in first-out; a failed allocation changes nothing.
#include <cstring>
#include <deque>
#include <unordered_map>
#include <vector>

#include "pkv_internal.h"

namespace {

struct Seq {
    std::vector<int32_t> table;  // device block ids, or host block ids while swapped out
    int32_t len = 0;
    bool swapped = false;
};

// One append, recorded so that a failed batch can be undone exactly.
struct Undo {
    int64_t seq;
    int32_t old_len;
    int32_t appended;  // block appended to the table, or -1
    int32_t cow_old;   // block replaced by a copy, or -1
    int32_t cow_new;
};

}  // namespace

struct pkv_bm {
    int32_t num_blocks = 0;
    int32_t block_size = 16;
    std::deque<int32_t> free_list;
    std::vector<int32_t> ref;
    std::unordered_map<int64_t, Seq> seqs;
    // host (swap) pool: blocks hold one swapped-out sequence's data each, never shared
    int32_t num_host_blocks = 0;
    std::deque<int32_t> host_free;

    int32_t take() {
        int32_t b = free_list.front();
        free_list.pop_front();
        ref[b] = 1;
        return b;
    }
    void untake(int32_t b) {
        ref[b] = 0;
        free_list.push_front(b);
    }

    // Append one token slot to s; returns false (and changes nothing) when out of blocks.
    bool append(int64_t id, Seq &s, int64_t *slot, int32_t *src, int32_t *dst, Undo *u) {
        const int32_t B = block_size;
        u->seq = id;
        u->old_len = s.len;
        u->appended = u->cow_old = u->cow_new = -1;
        *src = *dst = -1;
        if (s.len % B == 0) {
            if (free_list.empty()) return false;
            int32_t b = take();
            s.table.push_back(b);
            u->appended = b;
        } else {
            int32_t last = s.table.back();
            if (ref[last] > 1) {
                if (free_list.empty()) return false;
                int32_t b = take();
                ref[last] -= 1;
                s.table.back() = b;
                *src = last;
                *dst = b;
                u->cow_old = last;
                u->cow_new = b;
            }
        }
        *slot = (int64_t)s.table[s.len / B] * B + s.len % B;
        s.len += 1;
        return true;
    }

    void undo(const Undo &u) {
        Seq &s = seqs[u.seq];
        if (u.appended >= 0) {
            s.table.pop_back();
            untake(u.appended);
        }
        if (u.cow_old >= 0) {
            s.table.back() = u.cow_old;
            ref[u.cow_old] += 1;
            untake(u.cow_new);
        }
        s.len = u.old_len;
    }
};

using pkv::fail;

extern "C" {

pkv_status pkv_bm_create(int32_t num_blocks, int32_t block_size,
                         const int32_t *initial_free_order, pkv_bm **out) {
    if (!out) return fail(PKV_ERR_INVALID, "pkv_bm_create: out is NULL");
    *out = nullptr;
    if (num_blocks < 0) return fail(PKV_ERR_INVALID, "pkv_bm_create: num_blocks < 0");
    if (block_size != 16 && block_size != 32)
        return fail(PKV_ERR_UNSUPPORTED, "pkv_bm_create: block_size %d (16 or 32)", block_size);
    pkv_bm *bm = new (std::nothrow) pkv_bm;
    if (!bm) return fail(PKV_ERR_OOM, "pkv_bm_create: host allocation failed");
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->ref.assign(num_blocks, 0);
    if (initial_free_order) {
        std::vector<char> seen(num_blocks, 0);
        for (int32_t i = 0; i < num_blocks; ++i) {
            int32_t b = initial_free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete bm;
                return fail(PKV_ERR_INVALID,
                            "pkv_bm_create: initial_free_order is not a permutation");
            }
            seen[b] = 1;
            bm->free_list.push_back(b);
        }
    } else {
        for (int32_t i = 0; i < num_blocks; ++i) bm->free_list.push_back(i);
    }
    *out = bm;
    return PKV_OK;
}

void pkv_bm_destroy(pkv_bm *bm) { delete bm; }

pkv_status pkv_bm_add_seq(pkv_bm *bm, int64_t seq, int32_t num_tokens) {
    if (!bm) return fail(PKV_ERR_INVALID, "pkv_bm_add_seq: bm is NULL");
    if (num_tokens < 0) return fail(PKV_ERR_INVALID, "pkv_bm_add_seq: num_tokens < 0");
    if (bm->seqs.count(seq))
        return fail(PKV_ERR_INVALID, "pkv_bm_add_seq: sequence %lld exists", (long long)seq);
    int64_t need = ((int64_t)num_tokens + bm->block_size - 1) / bm->block_size;
    if (need > (int64_t)bm->free_list.size())
        return fail(PKV_ERR_OOM, "pkv_bm_add_seq: need %lld blocks, %zu free",
                    (long long)need, bm->free_list.size());
    Seq s;
    s.len = num_tokens;
    s.table.reserve(need);
    for (int64_t i = 0; i < need; ++i) s.table.push_back(bm->take());
    bm->seqs.emplace(seq, std::move(s));
    return PKV_OK;
}

pkv_status pkv_bm_append_slot(pkv_bm *bm, int64_t seq, int64_t *slot_out, int32_t *cow_src,
                              int32_t *cow_dst) {
    if (!bm || !slot_out || !cow_src || !cow_dst)
        return fail(PKV_ERR_INVALID, "pkv_bm_append_slot: NULL argument");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end())
        return fail(PKV_ERR_NOT_FOUND, "pkv_bm_append_slot: unknown sequence %lld",
                    (long long)seq);
    if (it->second.swapped)
        return fail(PKV_ERR_INVALID, "pkv_bm_append_slot: sequence %lld is swapped out",
                    (long long)seq);
    Undo u;
    if (!bm->append(seq, it->second, slot_out, cow_src, cow_dst, &u))
        return fail(PKV_ERR_OOM, "pkv_bm_append_slot: no free block");
    return PKV_OK;
}

pkv_status pkv_bm_append_slots(pkv_bm *bm, const int64_t *seqs, int32_t n, int64_t *slots_out,
                               int32_t *cow_pairs_out, int32_t *num_cow) {
    if (!bm || (n > 0 && (!seqs || !slots_out || !cow_pairs_out)) || !num_cow || n < 0)
        return fail(PKV_ERR_INVALID, "pkv_bm_append_slots: bad argument");
    *num_cow = 0;
    for (int32_t i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seqs[i]);
        if (it == bm->seqs.end())
            return fail(PKV_ERR_NOT_FOUND, "pkv_bm_append_slots: unknown sequence %lld",
                        (long long)seqs[i]);
        if (it->second.swapped)
            return fail(PKV_ERR_INVALID, "pkv_bm_append_slots: sequence %lld is swapped out",
                        (long long)seqs[i]);
    }
    std::vector<Undo> log((size_t)n);
    int32_t ncow = 0;
    for (int32_t i = 0; i < n; ++i) {
        int32_t src, dst;
        if (!bm->append(seqs[i], bm->seqs[seqs[i]], &slots_out[i], &src, &dst, &log[i])) {
            for (int32_t k = i - 1; k >= 0; --k) bm->undo(log[k]);
            return fail(PKV_ERR_OOM, "pkv_bm_append_slots: out of blocks at entry %d", i);
        }
        if (src >= 0) {
            cow_pairs_out[2 * ncow] = src;
            cow_pairs_out[2 * ncow + 1] = dst;
            ++ncow;
        }
    }
    *num_cow = ncow;
    return PKV_OK;
}

pkv_status pkv_bm_fork(pkv_bm *bm, int64_t parent, int64_t child) {
    if (!bm) return fail(PKV_ERR_INVALID, "pkv_bm_fork: bm is NULL");
    auto it = bm->seqs.find(parent);
    if (it == bm->seqs.end())
        return fail(PKV_ERR_NOT_FOUND, "pkv_bm_fork: unknown parent %lld", (long long)parent);
    if (bm->seqs.count(child))
        return fail(PKV_ERR_INVALID, "pkv_bm_fork: child %lld exists", (long long)child);
    if (it->second.swapped)
        return fail(PKV_ERR_INVALID, "pkv_bm_fork: parent %lld is swapped out",
                    (long long)parent);
    Seq c = it->second;
    for (int32_t b : c.table) bm->ref[b] += 1;
    bm->seqs.emplace(child, std::move(c));
    return PKV_OK;
}

pkv_status pkv_bm_free_seq(pkv_bm *bm, int64_t seq) {
    if (!bm) return fail(PKV_ERR_INVALID, "pkv_bm_free_seq: bm is NULL");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end())
        return fail(PKV_ERR_NOT_FOUND, "pkv_bm_free_seq: unknown sequence %lld",
                    (long long)seq);
    if (it->second.swapped) {
        for (int32_t b : it->second.table) bm->host_free.push_back(b);
    } else {
        for (int32_t b : it->second.table) {
            bm->ref[b] -= 1;
            if (bm->ref[b] == 0) bm->free_list.push_back(b);
        }
    }
    bm->seqs.erase(it);
    return PKV_OK;
}

pkv_status pkv_bm_block_table(const pkv_bm *bm, int64_t seq, int32_t *out, int32_t cap,
                              int32_t *n) {
    if (!bm || !n || (cap > 0 && !out))
        return fail(PKV_ERR_INVALID, "pkv_bm_block_table: bad argument");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end())
        return fail(PKV_ERR_NOT_FOUND, "pkv_bm_block_table: unknown sequence %lld",
                    (long long)seq);
    const std::vector<int32_t> &t = it->second.table;
    *n = (int32_t)t.size();
    int32_t m = cap < *n ? cap : *n;
    if (m > 0) std::memcpy(out, t.data(), sizeof(int32_t) * m);
    if (cap < *n) return fail(PKV_ERR_INVALID, "pkv_bm_block_table: capacity %d < %d", cap, *n);
    return PKV_OK;
}

pkv_status pkv_bm_block_tables(const pkv_bm *bm, const int64_t *seqs, int32_t n,
                               int32_t max_blocks, int32_t *out, int32_t *lens_out) {
    if (!bm || n < 0 || max_blocks < 0 || (n > 0 && (!seqs || !out || !lens_out)))
        return fail(PKV_ERR_INVALID, "pkv_bm_block_tables: bad argument");
    for (int32_t i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seqs[i]);
        if (it == bm->seqs.end())
            return fail(PKV_ERR_NOT_FOUND, "pkv_bm_block_tables: unknown sequence %lld",
                        (long long)seqs[i]);
        if (it->second.swapped)
            return fail(PKV_ERR_INVALID, "pkv_bm_block_tables: sequence %lld is swapped out",
                        (long long)seqs[i]);
        const std::vector<int32_t> &t = it->second.table;
        if ((int64_t)t.size() > max_blocks)
            return fail(PKV_ERR_INVALID, "pkv_bm_block_tables: sequence %lld has %zu blocks > %d",
                        (long long)seqs[i], t.size(), max_blocks);
        int32_t *row = out + (size_t)i * max_blocks;
        for (int32_t j = 0; j < max_blocks; ++j) row[j] = j < (int32_t)t.size() ? t[j] : -1;
        lens_out[i] = it->second.len;
    }
    return PKV_OK;
}

pkv_status pkv_bm_seq_len(const pkv_bm *bm, int64_t seq, int32_t *len) {
    if (!bm || !len) return fail(PKV_ERR_INVALID, "pkv_bm_seq_len: bad argument");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end())
        return fail(PKV_ERR_NOT_FOUND, "pkv_bm_seq_len: unknown sequence %lld", (long long)seq);
    *len = it->second.len;
    return PKV_OK;
}

pkv_status pkv_bm_refcount(const pkv_bm *bm, int32_t block, int32_t *count) {
    if (!bm || !count) return fail(PKV_ERR_INVALID, "pkv_bm_refcount: bad argument");
    if (block < 0 || block >= bm->num_blocks)
        return fail(PKV_ERR_INVALID, "pkv_bm_refcount: block %d out of range", block);
    *count = bm->ref[block];
    return PKV_OK;
}

pkv_status pkv_bm_set_host_pool(pkv_bm *bm, int32_t num_host_blocks,
                                const int32_t *initial_free_order) {
    if (!bm || num_host_blocks < 0)
        return fail(PKV_ERR_INVALID, "pkv_bm_set_host_pool: bad argument");
    for (auto &kv : bm->seqs)
        if (kv.second.swapped)
            return fail(PKV_ERR_INVALID, "pkv_bm_set_host_pool: sequences are swapped out");
    std::deque<int32_t> order;
    if (initial_free_order) {
        std::vector<char> seen(num_host_blocks, 0);
        for (int32_t i = 0; i < num_host_blocks; ++i) {
            int32_t b = initial_free_order[i];
            if (b < 0 || b >= num_host_blocks || seen[b])
                return fail(PKV_ERR_INVALID,
                            "pkv_bm_set_host_pool: initial_free_order is not a permutation");
            seen[b] = 1;
            order.push_back(b);
        }
    } else {
        for (int32_t i = 0; i < num_host_blocks; ++i) order.push_back(i);
    }
    bm->num_host_blocks = num_host_blocks;
    bm->host_free.swap(order);
    return PKV_OK;
}

pkv_status pkv_bm_swap_out(pkv_bm *bm, int64_t seq, int32_t *pairs_out, int32_t cap,
                           int32_t *n) {
    if (!bm || !n || (cap > 0 && !pairs_out))
        return fail(PKV_ERR_INVALID, "pkv_bm_swap_out: bad argument");
    *n = 0;
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end())
        return fail(PKV_ERR_NOT_FOUND, "pkv_bm_swap_out: unknown sequence %lld",
                    (long long)seq);
    Seq &s = it->second;
    if (s.swapped)
        return fail(PKV_ERR_INVALID, "pkv_bm_swap_out: sequence %lld is already swapped out",
                    (long long)seq);
    const int32_t nb = (int32_t)s.table.size();
    if (cap < nb) return fail(PKV_ERR_INVALID, "pkv_bm_swap_out: capacity %d < %d", cap, nb);
    if ((size_t)nb > bm->host_free.size())
        return fail(PKV_ERR_OOM, "pkv_bm_swap_out: need %d host blocks, %zu free", nb,
                    bm->host_free.size());
    for (int32_t j = 0; j < nb; ++j) {
        const int32_t g = s.table[j];
        const int32_t h = bm->host_free.front();
        bm->host_free.pop_front();
        pairs_out[2 * j] = g;
        pairs_out[2 * j + 1] = h;
        bm->ref[g] -= 1;
        if (bm->ref[g] == 0) bm->free_list.push_back(g);
        s.table[j] = h;
    }
    s.swapped = true;
    *n = nb;
    return PKV_OK;
}

pkv_status pkv_bm_swap_in(pkv_bm *bm, int64_t seq, int32_t *pairs_out, int32_t cap,
                          int32_t *n) {
    if (!bm || !n || (cap > 0 && !pairs_out))
        return fail(PKV_ERR_INVALID, "pkv_bm_swap_in: bad argument");
    *n = 0;
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end())
        return fail(PKV_ERR_NOT_FOUND, "pkv_bm_swap_in: unknown sequence %lld", (long long)seq);
    Seq &s = it->second;
    if (!s.swapped)
        return fail(PKV_ERR_INVALID, "pkv_bm_swap_in: sequence %lld is not swapped out",
                    (long long)seq);
    const int32_t nb = (int32_t)s.table.size();
    if (cap < nb) return fail(PKV_ERR_INVALID, "pkv_bm_swap_in: capacity %d < %d", cap, nb);
    if ((size_t)nb > bm->free_list.size())
        return fail(PKV_ERR_OOM, "pkv_bm_swap_in: need %d blocks, %zu free", nb,
                    bm->free_list.size());
    for (int32_t j = 0; j < nb; ++j) {
        const int32_t h = s.table[j];
        const int32_t g = bm->take();
        pairs_out[2 * j] = h;
        pairs_out[2 * j + 1] = g;
        bm->host_free.push_back(h);
        s.table[j] = g;
    }
    s.swapped = false;
    *n = nb;
    return PKV_OK;
}

pkv_status pkv_bm_is_swapped(const pkv_bm *bm, int64_t seq, int32_t *swapped) {
    if (!bm || !swapped) return fail(PKV_ERR_INVALID, "pkv_bm_is_swapped: bad argument");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end())
        return fail(PKV_ERR_NOT_FOUND, "pkv_bm_is_swapped: unknown sequence %lld",
                    (long long)seq);
    *swapped = it->second.swapped ? 1 : 0;
    return PKV_OK;
}

int32_t pkv_bm_num_host_free(const pkv_bm *bm) {
    return bm ? (int32_t)bm->host_free.size() : -1;
}

int32_t pkv_bm_num_free(const pkv_bm *bm) { return bm ? (int32_t)bm->free_list.size() : -1; }

int32_t pkv_bm_num_seqs(const pkv_bm *bm) { return bm ? (int32_t)bm->seqs.size() : -1; }

int32_t pkv_bm_free_list(const pkv_bm *bm, int32_t *out, int32_t cap) {
    if (!bm) return -1;
    int32_t i = 0;
    for (int32_t b : bm->free_list) {
        if (i < cap && out) out[i] = b;
        ++i;
    }
    return i;
}

}  // extern "C"
