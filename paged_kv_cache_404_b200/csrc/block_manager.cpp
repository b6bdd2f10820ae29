// block_manager.cpp -- host-side block manager of the paged KV cache.
//
// Decides where every token of every sequence goes:
//  - lazy allocation: a sequence receives a new block only when its last block
//    is full, from the front of the free list ("PagedAttention" glossary entry,
//    "Como funciona la paginacion" and its worked example, which pops blocks
//    [41, 7, 19] from the free list [41, 7, 19, 2, 33]); a prompt is allocated
//    first and its last block is then filled (iplexlaw.co.kr, logical vs
//    physical order);
//  - sharing: fork() makes a sequence that points at the same physical blocks,
//    counted per block (glossary entry, "Compartir bloques entre secuencias");
//  - copy-on-write: a sequence about to write into a partly filled block that
//    others still reference gets a fresh block and a (src, dst) copy request;
//    full shared blocks stay shared; the last holder writes in place
//    (iplexlaw.co.kr, "two answers to one request");
//  - release: a finished sequence drops its references and blocks whose count
//    reaches zero return to the back of the free list at once (glossary entry,
//    continuous batching);
//  - swap: a sequence's pages can move to a host pool and back, page by page,
//    instead of evicting whole sequences ("Le cache KV et PagedAttention",
//    fine-grained eviction); the manager decides the block pairs, the copies
//    run on the GPU (pkv_swap_blocks);
//  - prefix caching: full prompt blocks are registered under a key made of
//    their tokens and their parent block's key, so a later request whose
//    prompt starts the same way reuses them (glossary entry, full-block
//    hashing extends sharing across requests).  A registered block that no
//    sequence uses stays in the free list with its contents; a hit takes it
//    back out, and reusing it for new data drops its registration.
// Plain C++ with host memory only; exported through the C ABI in pagedkv.h.
#include <cstdint>
#include <cstring>
#include <deque>
#include <functional>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

// Key of a full prompt block: the registration serial of its parent block (0
// for a prompt's first block), then its block_size token ids.  Exact content,
// hashed only to find the bucket, so two different prefixes never share a key.
struct KeyHash {
    size_t operator()(const std::vector<int64_t>& k) const {
        uint64_t h = 1469598103934665603ull;
        for (int64_t x : k) {
            h ^= (uint64_t)x;
            h *= 1099511628211ull;
            h ^= h >> 29;
        }
        return (size_t)h;
    }
};

struct CachedBlock {
    int32_t block;
    uint64_t serial;  // unique per registration: children are keyed by it
};

struct pkv_block_manager {
    int num_blocks = 0;
    int block_size = 0;
    // Free list, first in first out.  An entry is live while its block is free
    // and its generation matches; a cached block taken back out of the list
    // leaves a dead entry behind (skipped when it reaches the front).
    std::deque<std::pair<int32_t, uint32_t>> free_q;
    std::vector<uint32_t> free_gen;
    std::vector<uint8_t> is_free;
    size_t free_count = 0;
    std::vector<int32_t> refs;                  // per physical block
    std::vector<std::vector<int32_t>> tables;   // per sequence id
    std::vector<int32_t> lens;                  // tokens per sequence
    std::vector<uint8_t> alive;
    std::vector<uint8_t> swapped;               // table holds host block ids
    int num_host_blocks = 0;
    std::deque<int32_t> host_free;
    std::vector<uint8_t> host_used;
    bool prefix_cache = false;
    uint64_t next_serial = 1;
    std::unordered_map<std::vector<int64_t>, CachedBlock, KeyHash> cache;
    std::vector<std::vector<int64_t>> key_of;  // per block: its key, empty if unregistered

    bool valid_seq(int32_t s) const { return s >= 0 && (size_t)s < tables.size() && alive[s]; }
    // resident (on the device) sequence: PKV_OK, else the error to return
    int resident(int32_t s) const {
        if (!valid_seq(s)) return PKV_ENOENT;
        return swapped[s] ? PKV_ESWAPPED : PKV_OK;
    }

    void push_free(int32_t b) {
        is_free[b] = 1;
        free_q.emplace_back(b, ++free_gen[b]);
        ++free_count;
    }

    // a cached free block reused by a hit: its queue entry goes dead
    void revive(int32_t b) {
        is_free[b] = 0;
        --free_count;
        refs[b] = 1;
    }

    void uncache(int32_t b) {
        if (!key_of.empty() && !key_of[b].empty()) {
            cache.erase(key_of[b]);
            key_of[b].clear();
        }
    }

    int32_t take_block() {
        for (;;) {
            const std::pair<int32_t, uint32_t> e = free_q.front();
            free_q.pop_front();
            if (is_free[e.first] && free_gen[e.first] == e.second) {
                const int32_t b = e.first;
                is_free[b] = 0;
                --free_count;
                uncache(b);  // new contents: the old key no longer describes it
                refs[b] = 1;
                return b;
            }
        }
    }

    void release(int32_t b) {
        if (--refs[b] == 0) push_free(b);
    }

    int32_t new_seq(std::vector<int32_t>&& table, int32_t len) {
        tables.push_back(std::move(table));
        lens.push_back(len);
        alive.push_back(1);
        swapped.push_back(0);
        return (int32_t)(tables.size() - 1);
    }
};

extern "C" {

int pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order, int free_count,
                  pkv_block_manager** out) {
    if (out == nullptr || num_blocks <= 0 || block_size <= 0) return PKV_EINVAL;
    pkv_block_manager* bm = new (std::nothrow) pkv_block_manager();
    if (bm == nullptr) return PKV_ENOMEM;
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->refs.assign(num_blocks, 0);
    bm->free_gen.assign(num_blocks, 0);
    bm->is_free.assign(num_blocks, 0);
    if (free_order == nullptr) {
        for (int b = 0; b < num_blocks; ++b) bm->push_free(b);
    } else {
        std::vector<uint8_t> seen(num_blocks, 0);
        for (int i = 0; i < free_count; ++i) {
            const int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete bm;
                return PKV_EINVAL;
            }
            seen[b] = 1;
            bm->push_free(b);
        }
    }
    *out = bm;
    return PKV_OK;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

int pkv_bm_alloc_seq(pkv_block_manager* bm, int num_tokens, int32_t* seq_out) {
    if (bm == nullptr || seq_out == nullptr || num_tokens < 0) return PKV_EINVAL;
    const size_t need = ((size_t)num_tokens + bm->block_size - 1) / bm->block_size;
    if (need > bm->free_count) return PKV_ENOMEM;
    std::vector<int32_t> table;
    table.reserve(need);
    for (size_t i = 0; i < need; ++i) table.push_back(bm->take_block());
    *seq_out = bm->new_seq(std::move(table), num_tokens);
    return PKV_OK;
}

int pkv_bm_fork(pkv_block_manager* bm, int32_t parent, int32_t* child_out) {
    if (bm == nullptr || child_out == nullptr) return PKV_EINVAL;
    if (int st = bm->resident(parent)) return st;
    std::vector<int32_t> table = bm->tables[parent];
    for (int32_t b : table) ++bm->refs[b];
    *child_out = bm->new_seq(std::move(table), bm->lens[parent]);
    return PKV_OK;
}

int pkv_bm_fork_many(pkv_block_manager* bm, const int32_t* parents, int n, int32_t* children_out) {
    if (bm == nullptr || n < 0 || (n > 0 && (parents == nullptr || children_out == nullptr))) return PKV_EINVAL;
    for (int i = 0; i < n; ++i)
        if (int st = bm->resident(parents[i])) return st;  // checked first: nothing changes on error
    for (int i = 0; i < n; ++i) {
        int st = pkv_bm_fork(bm, parents[i], &children_out[i]);
        if (st != PKV_OK) return st;
    }
    return PKV_OK;
}

int pkv_bm_free_many(pkv_block_manager* bm, const int32_t* seqs, int n) {
    if (bm == nullptr || n < 0 || (n > 0 && seqs == nullptr)) return PKV_EINVAL;
    for (int i = 0; i < n; ++i) {
        if (!bm->valid_seq(seqs[i])) return PKV_ENOENT;
        for (int j = 0; j < i; ++j)
            if (seqs[j] == seqs[i]) return PKV_EINVAL;  // a sequence listed twice
    }
    for (int i = 0; i < n; ++i) pkv_bm_free_seq(bm, seqs[i]);
    return PKV_OK;
}

int pkv_bm_append_tokens(pkv_block_manager* bm, const int32_t* seqs, int n, int64_t* slots_out,
                         int64_t* cow_pairs_out, int* num_pairs_out, int* num_done_out) {
    if (bm == nullptr || n < 0 || (n > 0 && (seqs == nullptr || slots_out == nullptr || cow_pairs_out == nullptr)))
        return PKV_EINVAL;
    int pairs = 0;
    int done = 0;
    int status = PKV_OK;
    for (; done < n; ++done) {
        const int32_t s = seqs[done];
        if (int st = bm->resident(s)) {
            status = st;
            break;
        }
        std::vector<int32_t>& table = bm->tables[s];
        const int32_t len = bm->lens[s];
        const int32_t off = len % bm->block_size;
        if (off == 0) {
            // last block full (or none yet): next free block, nothing to copy
            if (bm->free_count == 0) {
                status = PKV_ENOMEM;
                break;
            }
            table.push_back(bm->take_block());
        } else if (bm->refs[table.back()] > 1) {
            // partly filled block still shared: copy it, write into the copy
            if (bm->free_count == 0) {
                status = PKV_ENOMEM;
                break;
            }
            const int32_t src = table.back();
            const int32_t dst = bm->take_block();
            --bm->refs[src];
            table.back() = dst;
            cow_pairs_out[2 * pairs] = src;
            cow_pairs_out[2 * pairs + 1] = dst;
            ++pairs;
        }
        slots_out[done] = (int64_t)table[len / bm->block_size] * bm->block_size + off;
        bm->lens[s] = len + 1;
    }
    if (num_pairs_out) *num_pairs_out = pairs;
    if (num_done_out) *num_done_out = done;
    return status;
}

int pkv_bm_free_seq(pkv_block_manager* bm, int32_t seq) {
    if (bm == nullptr) return PKV_EINVAL;
    if (!bm->valid_seq(seq)) return PKV_ENOENT;
    if (bm->swapped[seq]) {
        for (int32_t h : bm->tables[seq]) {
            bm->host_used[h] = 0;
            bm->host_free.push_back(h);
        }
    } else {
        for (int32_t b : bm->tables[seq]) {
            bm->release(b);
        }
    }
    bm->tables[seq].clear();
    bm->tables[seq].shrink_to_fit();
    bm->lens[seq] = 0;
    bm->alive[seq] = 0;
    bm->swapped[seq] = 0;
    return PKV_OK;
}

int pkv_bm_num_free(const pkv_block_manager* bm) { return bm ? (int)bm->free_count : -1; }

int pkv_bm_seq_len(const pkv_block_manager* bm, int32_t seq, int32_t* len_out) {
    if (bm == nullptr || len_out == nullptr) return PKV_EINVAL;
    if (!bm->valid_seq(seq)) return PKV_ENOENT;
    *len_out = bm->lens[seq];
    return PKV_OK;
}

int pkv_bm_refcount(const pkv_block_manager* bm, int32_t block, int32_t* rc_out) {
    if (bm == nullptr || rc_out == nullptr || block < 0 || block >= bm->num_blocks) return PKV_EINVAL;
    *rc_out = bm->refs[block];
    return PKV_OK;
}

int pkv_bm_block_table(const pkv_block_manager* bm, int32_t seq, int32_t* out, int cap, int* n_out) {
    if (bm == nullptr || n_out == nullptr || cap < 0 || (cap > 0 && out == nullptr)) return PKV_EINVAL;
    if (!bm->valid_seq(seq)) return PKV_ENOENT;
    const std::vector<int32_t>& t = bm->tables[seq];
    *n_out = (int)t.size();
    if ((int)t.size() > cap) return PKV_EINVAL;
    if (!t.empty()) std::memcpy(out, t.data(), t.size() * sizeof(int32_t));
    return PKV_OK;
}

int pkv_bm_slots(const pkv_block_manager* bm, int32_t seq, int start, int count, int64_t* out) {
    if (bm == nullptr || start < 0 || count < 0 || (count > 0 && out == nullptr)) return PKV_EINVAL;
    if (int st = bm->resident(seq)) return st;
    const std::vector<int32_t>& t = bm->tables[seq];
    if ((size_t)start + count > t.size() * (size_t)bm->block_size) return PKV_EINVAL;
    for (int i = 0; i < count; ++i) {
        const int pos = start + i;
        out[i] = (int64_t)t[pos / bm->block_size] * bm->block_size + pos % bm->block_size;
    }
    return PKV_OK;
}

int pkv_bm_tables(const pkv_block_manager* bm, const int32_t* seqs, int n, int32_t* tables, int max_blocks,
                  int32_t pad, int32_t* lens) {
    if (bm == nullptr || n < 0 || max_blocks <= 0 || (n > 0 && (seqs == nullptr || tables == nullptr)))
        return PKV_EINVAL;
    for (int i = 0; i < n; ++i) {
        if (int st = bm->resident(seqs[i])) return st;
        const std::vector<int32_t>& t = bm->tables[seqs[i]];
        if ((int)t.size() > max_blocks) return PKV_EINVAL;
        int32_t* row = tables + (size_t)i * max_blocks;
        for (int j = 0; j < max_blocks; ++j) row[j] = j < (int)t.size() ? t[j] : pad;
        if (lens) lens[i] = bm->lens[seqs[i]];
    }
    return PKV_OK;
}

int pkv_bm_free_list(const pkv_block_manager* bm, int32_t* out, int cap, int* n_out) {
    if (bm == nullptr || n_out == nullptr || cap < 0 || (cap > 0 && out == nullptr)) return PKV_EINVAL;
    *n_out = (int)bm->free_count;
    if ((int)bm->free_count > cap) return PKV_EINVAL;
    int i = 0;
    for (const std::pair<int32_t, uint32_t>& e : bm->free_q)
        if (bm->is_free[e.first] && bm->free_gen[e.first] == e.second) out[i++] = e.first;
    return PKV_OK;
}

int pkv_bm_prefix_groups(const pkv_block_manager* bm, const int32_t* seqs, int n, int32_t* group_offsets,
                         int32_t* group_seqs, int32_t* group_shared_blocks, int* num_groups_out) {
    if (bm == nullptr || n < 0 || num_groups_out == nullptr ||
        (n > 0 && (seqs == nullptr || group_offsets == nullptr || group_seqs == nullptr ||
                   group_shared_blocks == nullptr)))
        return PKV_EINVAL;
    for (int i = 0; i < n; ++i)
        if (int st = bm->resident(seqs[i])) return st;
    // batch indices grouped by the physical id of their first block
    std::unordered_map<int32_t, int> by_first;
    std::vector<std::vector<int>> groups;
    for (int i = 0; i < n; ++i) {
        if (bm->lens[seqs[i]] < bm->block_size) continue;  // no full block
        const int32_t b0 = bm->tables[seqs[i]][0];
        auto it = by_first.find(b0);
        if (it == by_first.end()) {
            by_first.emplace(b0, (int)groups.size());
            groups.push_back({i});
        } else {
            groups[it->second].push_back(i);
        }
    }
    int ng = 0, pos = 0;
    if (n > 0) group_offsets[0] = 0;
    for (const std::vector<int>& g : groups) {
        if (g.size() < 2) continue;
        const std::vector<int32_t>& t0 = bm->tables[seqs[g[0]]];
        int k = bm->lens[seqs[g[0]]] / bm->block_size;
        for (int m : g) {
            const std::vector<int32_t>& tm = bm->tables[seqs[m]];
            const int full = bm->lens[seqs[m]] / bm->block_size;
            if (full < k) k = full;
            int j = 0;
            while (j < k && tm[j] == t0[j]) ++j;
            k = j;
        }
        for (int m : g) group_seqs[pos++] = m;
        group_shared_blocks[ng++] = k;
        group_offsets[ng] = pos;
    }
    *num_groups_out = ng;
    return PKV_OK;
}

int pkv_bm_set_prefix_cache(pkv_block_manager* bm, int enable) {
    if (bm == nullptr) return PKV_EINVAL;
    bm->prefix_cache = enable != 0;
    if (!bm->prefix_cache) {
        bm->cache.clear();
        bm->key_of.clear();
    } else if (bm->key_of.empty()) {
        bm->key_of.assign(bm->num_blocks, {});
    }
    return PKV_OK;
}

int pkv_bm_alloc_seq_tokens(pkv_block_manager* bm, const int32_t* tokens, int num_tokens, int32_t* seq_out,
                            int* num_cached_out) {
    if (bm == nullptr || seq_out == nullptr || num_tokens < 0 || (num_tokens > 0 && tokens == nullptr))
        return PKV_EINVAL;
    if (!bm->prefix_cache) {
        if (num_cached_out) *num_cached_out = 0;
        return pkv_bm_alloc_seq(bm, num_tokens, seq_out);
    }
    const int bs = bm->block_size;
    const int full = num_tokens / bs;
    const size_t need = ((size_t)num_tokens + bs - 1) / bs;
    auto key = [&](uint64_t parent, int j) {
        std::vector<int64_t> k;
        k.reserve(bs + 1);
        k.push_back((int64_t)parent);
        for (int i = 0; i < bs; ++i) k.push_back(tokens[(size_t)j * bs + i]);
        return k;
    };
    // 1. longest run of leading full blocks already registered
    std::vector<CachedBlock> hits;
    uint64_t parent = 0;
    for (int j = 0; j < full; ++j) {
        auto it = bm->cache.find(key(parent, j));
        if (it == bm->cache.end()) break;
        hits.push_back(it->second);
        parent = it->second.serial;
    }
    size_t revived = 0;
    for (const CachedBlock& h : hits) revived += bm->refs[h.block] == 0;
    if (need - hits.size() + revived > bm->free_count) return PKV_ENOMEM;
    // 2. take the hits (shared, or back out of the free list), then new blocks
    std::vector<int32_t> table;
    table.reserve(need);
    for (const CachedBlock& h : hits) {
        if (bm->refs[h.block] == 0)
            bm->revive(h.block);
        else
            ++bm->refs[h.block];
        table.push_back(h.block);
    }
    while (table.size() < need) table.push_back(bm->take_block());
    // 3. register the new full blocks, each keyed by its parent's serial
    for (int j = (int)hits.size(); j < full; ++j) {
        std::vector<int64_t> k = key(parent, j);
        const CachedBlock c{table[j], bm->next_serial++};
        bm->key_of[c.block] = k;
        bm->cache.emplace(std::move(k), c);
        parent = c.serial;
    }
    if (num_cached_out) *num_cached_out = (int)hits.size() * bs;
    *seq_out = bm->new_seq(std::move(table), num_tokens);
    return PKV_OK;
}

int pkv_bm_num_cached_blocks(const pkv_block_manager* bm) { return bm ? (int)bm->cache.size() : -1; }

int pkv_bm_set_host_pool(pkv_block_manager* bm, int num_host_blocks) {
    if (bm == nullptr || num_host_blocks < 0) return PKV_EINVAL;
    for (uint8_t u : bm->host_used)
        if (u) return PKV_EINVAL;  // host blocks still hold swapped pages
    bm->num_host_blocks = num_host_blocks;
    bm->host_used.assign(num_host_blocks, 0);
    bm->host_free.clear();
    for (int h = 0; h < num_host_blocks; ++h) bm->host_free.push_back(h);
    return PKV_OK;
}

int pkv_bm_swap_out(pkv_block_manager* bm, int32_t seq, int64_t* pairs_out, int cap, int* num_pairs_out) {
    if (bm == nullptr || num_pairs_out == nullptr || cap < 0) return PKV_EINVAL;
    if (int st = bm->resident(seq)) return st;
    std::vector<int32_t>& table = bm->tables[seq];
    const int k = (int)table.size();
    *num_pairs_out = 0;
    if (k > cap || (k > 0 && pairs_out == nullptr)) return PKV_EINVAL;
    if ((size_t)k > bm->host_free.size()) return PKV_ENOMEM;
    for (int i = 0; i < k; ++i) {
        const int32_t h = bm->host_free.front();
        bm->host_free.pop_front();
        bm->host_used[h] = 1;
        const int32_t d = table[i];
        pairs_out[2 * i] = d;
        pairs_out[2 * i + 1] = h;
        // a page another sequence still uses stays on the device
        bm->release(d);
        table[i] = h;
    }
    bm->swapped[seq] = 1;
    *num_pairs_out = k;
    return PKV_OK;
}

int pkv_bm_swap_in(pkv_block_manager* bm, int32_t seq, int64_t* pairs_out, int cap, int* num_pairs_out) {
    if (bm == nullptr || num_pairs_out == nullptr || cap < 0) return PKV_EINVAL;
    if (!bm->valid_seq(seq)) return PKV_ENOENT;
    if (!bm->swapped[seq]) return PKV_EINVAL;
    std::vector<int32_t>& table = bm->tables[seq];
    const int k = (int)table.size();
    *num_pairs_out = 0;
    if (k > cap || (k > 0 && pairs_out == nullptr)) return PKV_EINVAL;
    if ((size_t)k > bm->free_count) return PKV_ENOMEM;
    for (int i = 0; i < k; ++i) {
        const int32_t h = table[i];
        const int32_t d = bm->take_block();
        pairs_out[2 * i] = h;
        pairs_out[2 * i + 1] = d;
        bm->host_used[h] = 0;
        bm->host_free.push_back(h);
        table[i] = d;
    }
    bm->swapped[seq] = 0;
    *num_pairs_out = k;
    return PKV_OK;
}

int pkv_bm_is_swapped(const pkv_block_manager* bm, int32_t seq, int* swapped_out) {
    if (bm == nullptr || swapped_out == nullptr) return PKV_EINVAL;
    if (!bm->valid_seq(seq)) return PKV_ENOENT;
    *swapped_out = bm->swapped[seq];
    return PKV_OK;
}

int pkv_bm_num_free_host(const pkv_block_manager* bm) { return bm ? (int)bm->host_free.size() : -1; }

}  // extern "C"
