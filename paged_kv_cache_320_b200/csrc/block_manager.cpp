// Host KV block manager: free list, reference counts, fork, copy-on-write.
//
// "vLLM" entity page, 是什么: blocks are handed out only when a sequence needs one,
// the last block is the only partly empty one, and sampled continuations / common
// prompts share physical blocks through reference counts and copy-on-write.
// "vLLM / PagedAttention — 分页 KV Cache 分析" §2.3 (a global page allocator and one
// block table per request), §3.2 (copy a shared page before changing it) and §3.3
// (finished requests give their pages back at once).
//
// The order rules the pages leave open are stated in pagedkv.h (LIFO free list
// seeded by initial_order, free walks a table from its last block, all-or-nothing
// appends). Pure host code: no CUDA call.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <list>
#include <memory>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

namespace {

// splitmix64 (Steele, Lea, Flood: "Fast splittable pseudorandom number generators",
// OOPSLA 2014), used as a mixing function for the prefix hash chain.
uint64_t splitmix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// Hash of a full block given the hash of everything before it (0 for the first).
uint64_t chain_hash(uint64_t parent, const int32_t *tokens, int n) {
    uint64_t h = parent;
    for (int i = 0; i < n; ++i) h = splitmix64(h ^ (uint64_t)(uint32_t)tokens[i]);
    return h;
}

struct Seq {
    std::vector<int32_t> table;  // logical block -> physical block
    int64_t len = 0;             // tokens written
    // prefix caching: token ids of the partly filled last block and the chain hash of
    // the full blocks before it; `tracked` = every token so far came with its id
    bool tracked = false;
    uint64_t hash = 0;
    std::vector<int32_t> partial;
};

struct CachedBlock {
    uint64_t parent;              // chain hash of the blocks before it
    std::vector<int32_t> tokens;  // its block_size token ids
    int32_t block;
};

// Runs f, turning any exception (a failed host allocation: std::bad_alloc, or a
// container grown past its maximum size) into PKV_ERR_HOST_MEMORY, so that nothing
// throws across the C ABI.
template <class F>
int guarded(F &&f) noexcept {
    try {
        return f();
    } catch (...) {
        return PKV_ERR_HOST_MEMORY;
    }
}

}  // namespace

struct pkv_alloc {
    int num_blocks = 0;
    int block_size = 0;
    int max_blocks = 0;
    std::vector<int32_t> free_stack;  // back() is the next block handed out
    std::vector<int32_t> refcount;
    // sequence records: a freed record's slot is reused with its vectors' capacity, so a
    // steady fork / free cycle allocates no table memory
    std::vector<Seq> pool;
    std::vector<int32_t> free_slots;
    std::unordered_map<int64_t, int32_t> index;   // sequence id -> slot in pool
    int64_t logical_tokens = 0;
    // prefix cache: chain hash -> cached block; blocks whose count fell to 0 while cached
    // wait, least recently released first, in `evictable` until a free block is needed
    bool prefix_cache = false;
    std::unordered_map<uint64_t, CachedBlock> cache;
    std::vector<uint64_t> block_key;   // per block: its cache key (valid if cached[b])
    std::vector<char> cached;
    std::list<int32_t> evictable;
    std::vector<std::list<int32_t>::iterator> evict_pos;
    int64_t query_tokens = 0, hit_tokens = 0;

    int available() const { return (int)(free_stack.size() + evictable.size()); }

    Seq *find(int64_t id) {
        auto it = index.find(id);
        return it == index.end() ? nullptr : &pool[it->second];
    }
    const Seq *find(int64_t id) const {
        auto it = index.find(id);
        return it == index.end() ? nullptr : &pool[it->second];
    }

    // An empty record for an id not in use; returns its slot. Growing the pool may move
    // records: hold slots, not references, across this call.
    int32_t add(int64_t id) {
        int32_t slot;
        if (!free_slots.empty()) {
            slot = free_slots.back();
            free_slots.pop_back();
        } else {
            slot = (int32_t)pool.size();
            pool.emplace_back();
        }
        Seq &s = pool[slot];
        s.table.clear();
        s.len = 0;
        s.tracked = false;
        s.hash = 0;
        s.partial.clear();
        index.emplace(id, slot);
        return slot;
    }

    int32_t take() {
        int32_t b;
        if (!free_stack.empty()) {
            b = free_stack.back();
            free_stack.pop_back();
        } else {
            // reclaim the least recently released cached block: its contents go
            b = evictable.front();
            evictable.pop_front();
            cache.erase(block_key[b]);
            cached[b] = 0;
        }
        refcount[b] = 1;
        return b;
    }

    // one reference fewer; a block nobody holds is freed, or kept for reuse if cached
    void release(int32_t b) {
        if (--refcount[b] != 0) return;
        if (cached[b]) {
            evictable.push_back(b);
            evict_pos[b] = std::prev(evictable.end());
        } else {
            free_stack.push_back(b);
        }
    }

    // a new holder of cached block b (from the prefix cache)
    void acquire_cached(int32_t b) {
        if (refcount[b] == 0) evictable.erase(evict_pos[b]);
        refcount[b] += 1;
    }

    // the token at position n of s (already placed) completes or extends its block
    void record_token(Seq &s, int64_t n, const int32_t *token) {
        if (!prefix_cache || !s.tracked) return;
        if (!token) {
            s.tracked = false;   // an id is missing: this sequence stops sharing
            s.partial.clear();
            return;
        }
        s.partial.push_back(*token);
        if ((int)s.partial.size() < block_size) return;
        const uint64_t key = chain_hash(s.hash, s.partial.data(), block_size);
        const int32_t b = s.table[n / block_size];
        if (!cache.count(key) && !cached[b]) {
            cache.emplace(key, CachedBlock{s.hash, s.partial, b});
            block_key[b] = key;
            cached[b] = 1;
        }
        s.hash = key;
        s.partial.clear();
    }

    // Blocks an append of n tokens to `s` (nullptr = new sequence) would take.
    void needs(const Seq *s, int n, int64_t *blocks, int64_t *table_len) const {
        const int64_t len = s ? s->len : 0;
        int64_t need = 0;
        if (n > 0 && s && len % block_size != 0 && !s->table.empty() &&
            refcount[s->table.back()] > 1)
            need += 1;  // copy-on-write of the shared partial last block
        // positions p in [len, len + n) with p % bs == 0 start a new block
        const int64_t first_new = (len + block_size - 1) / block_size;
        const int64_t last_needed = (len + n + block_size - 1) / block_size;
        need += std::max<int64_t>(0, last_needed - first_new);
        *blocks = need;
        *table_len = last_needed;
    }
};

extern "C" {

int pkv_alloc_create(pkv_alloc **out, int num_blocks, int block_size, int max_blocks_per_seq,
                     const int32_t *initial_order) {
    return guarded([&]() -> int {
        if (!out || num_blocks <= 0 || block_size <= 0 || max_blocks_per_seq <= 0)
            return PKV_ERR_INVALID_ARG;
        *out = nullptr;
        std::vector<char> seen(num_blocks, 0);
        if (initial_order) {
            for (int i = 0; i < num_blocks; ++i) {
                const int32_t b = initial_order[i];
                if (b < 0 || b >= num_blocks || seen[b]) return PKV_ERR_INVALID_ARG;
                seen[b] = 1;
            }
        }
        std::unique_ptr<pkv_alloc> a(new (std::nothrow) pkv_alloc());
        if (!a) return PKV_ERR_HOST_MEMORY;
        a->num_blocks = num_blocks;
        a->block_size = block_size;
        a->max_blocks = max_blocks_per_seq;
        a->refcount.assign(num_blocks, 0);
        a->block_key.assign(num_blocks, 0);
        a->cached.assign(num_blocks, 0);
        a->evict_pos.resize(num_blocks);
        a->free_stack.resize(num_blocks);
        for (int i = 0; i < num_blocks; ++i)
            a->free_stack[num_blocks - 1 - i] = initial_order ? initial_order[i] : i;
        *out = a.release();
        return PKV_OK;
    });
}

int pkv_alloc_destroy(pkv_alloc *a) {
    delete a;
    return PKV_OK;
}

namespace {

// tokens == nullptr: an append without ids (with_ids false)
int append_impl(pkv_alloc *a, int64_t seq_id, int n_tokens, bool with_ids, const int32_t *tokens,
                int64_t *slots_out, int32_t *cow_pairs_out, int *n_cow_out) {
    if (!a || n_tokens < 0) return PKV_ERR_INVALID_ARG;
    if (n_tokens > 0 && !slots_out) return PKV_ERR_INVALID_ARG;
    const Seq *existing = a->find(seq_id);
    int64_t need, table_len;
    a->needs(existing, n_tokens, &need, &table_len);
    if (table_len > a->max_blocks) return PKV_ERR_TABLE_FULL;
    if (need > (int64_t)a->available()) return PKV_ERR_OUT_OF_BLOCKS;
    if (need > 0 && !cow_pairs_out && existing && existing->len % a->block_size != 0 &&
        a->refcount[existing->table.back()] > 1)
        return PKV_ERR_INVALID_ARG;  // a copy-on-write pair would be lost
    const bool created = !existing;
    Seq &s = created ? a->pool[a->add(seq_id)] : *a->find(seq_id);
    if (created) s.tracked = a->prefix_cache && with_ids;
    const int bs = a->block_size;
    int n_cow = 0;
    for (int i = 0; i < n_tokens; ++i) {
        const int64_t n = s.len;
        if (n % bs == 0) {
            s.table.push_back(a->take());
        } else if (a->refcount[s.table.back()] > 1) {
            const int32_t old = s.table.back();
            const int32_t fresh = a->take();
            cow_pairs_out[2 * n_cow] = old;
            cow_pairs_out[2 * n_cow + 1] = fresh;
            ++n_cow;
            a->refcount[old] -= 1;
            s.table.back() = fresh;
        }
        slots_out[i] = (int64_t)s.table[n / bs] * bs + n % bs;
        s.len = n + 1;
        a->record_token(s, n, with_ids ? tokens + i : nullptr);
    }
    a->logical_tokens += n_tokens;
    if (n_cow_out) *n_cow_out = n_cow;
    return PKV_OK;
}

}  // namespace

int pkv_seq_append(pkv_alloc *a, int64_t seq_id, int n_tokens, int64_t *slots_out,
                   int32_t *cow_pairs_out, int *n_cow_out) {
    return guarded([&]() -> int {
        return append_impl(a, seq_id, n_tokens, false, nullptr, slots_out, cow_pairs_out, n_cow_out);
    });
}

int pkv_seq_append_tokens(pkv_alloc *a, int64_t seq_id, const int32_t *tokens, int n_tokens,
                          int64_t *slots_out, int32_t *cow_pairs_out, int *n_cow_out) {
    return guarded([&]() -> int {
        if (n_tokens > 0 && !tokens) return PKV_ERR_INVALID_ARG;
        return append_impl(a, seq_id, n_tokens, true, tokens, slots_out, cow_pairs_out, n_cow_out);
    });
}

int pkv_alloc_set_prefix_cache(pkv_alloc *a, int enable) {
    return guarded([&]() -> int {
        if (!a || (enable != 0 && enable != 1)) return PKV_ERR_INVALID_ARG;
        if (a->prefix_cache && !enable) {
            // forget every cached block; the ones nobody holds become free
            for (int32_t b : a->evictable) a->free_stack.push_back(b);
            a->evictable.clear();
            a->cache.clear();
            std::fill(a->cached.begin(), a->cached.end(), 0);
            for (auto &kv : a->index) {
                a->pool[kv.second].tracked = false;
                a->pool[kv.second].partial.clear();
            }
        }
        a->prefix_cache = enable != 0;
        return PKV_OK;
    });
}

int pkv_seq_share_prefix(pkv_alloc *a, int64_t seq_id, const int32_t *tokens, int n_tokens,
                         int *n_cached_out) {
    return guarded([&]() -> int {
        if (!a || n_tokens < 0 || (n_tokens > 0 && !tokens)) return PKV_ERR_INVALID_ARG;
        if (a->index.count(seq_id)) return PKV_ERR_SEQ_EXISTS;
        Seq s;
        s.tracked = a->prefix_cache;
        const int bs = a->block_size;
        int matched = 0;
        if (a->prefix_cache) {
            for (int j = 0; (j + 1) * bs <= n_tokens && j < a->max_blocks; ++j) {
                const int32_t *blk = tokens + (size_t)j * bs;
                const uint64_t key = chain_hash(s.hash, blk, bs);
                auto hit = a->cache.find(key);
                if (hit == a->cache.end() || hit->second.parent != s.hash ||
                    std::memcmp(hit->second.tokens.data(), blk, sizeof(int32_t) * bs) != 0)
                    break;
                a->acquire_cached(hit->second.block);
                s.table.push_back(hit->second.block);
                s.hash = key;
                matched += bs;
            }
            a->query_tokens += n_tokens;
            a->hit_tokens += matched;
        }
        s.len = matched;
        a->logical_tokens += matched;
        a->pool[a->add(seq_id)] = std::move(s);
        if (n_cached_out) *n_cached_out = matched;
        return PKV_OK;
    });
}

int pkv_prefix_cache_stats(const pkv_alloc *a, int *cached_blocks, int *evictable_blocks,
                           int64_t *query_tokens, int64_t *hit_tokens) {
    if (!a) return PKV_ERR_INVALID_ARG;
    if (cached_blocks) *cached_blocks = (int)a->cache.size();
    if (evictable_blocks) *evictable_blocks = (int)a->evictable.size();
    if (query_tokens) *query_tokens = a->query_tokens;
    if (hit_tokens) *hit_tokens = a->hit_tokens;
    return PKV_OK;
}

int pkv_seq_append_batch(pkv_alloc *a, const int64_t *seq_ids, int n, int n_tokens,
                         int64_t *slots_out, int32_t *cow_pairs_out, int *n_cow_out,
                         int *n_done_out) {
    if (n_done_out) *n_done_out = 0;
    if (n_cow_out) *n_cow_out = 0;
    if (!a || n < 0 || n_tokens < 0 || (n > 0 && !seq_ids)) return PKV_ERR_INVALID_ARG;
    if (n > 0 && n_tokens > 0 && (!slots_out || !cow_pairs_out)) return PKV_ERR_INVALID_ARG;
    int total_cow = 0;
    for (int i = 0; i < n; ++i) {
        int k = 0;
        const int rc = pkv_seq_append(a, seq_ids[i], n_tokens,
                                      slots_out ? slots_out + (size_t)i * n_tokens : nullptr,
                                      cow_pairs_out ? cow_pairs_out + 2 * (size_t)total_cow
                                                    : nullptr,
                                      &k);
        if (rc != PKV_OK) {
            if (n_cow_out) *n_cow_out = total_cow;
            return rc;
        }
        total_cow += k;
        if (n_done_out) *n_done_out = i + 1;
    }
    if (n_cow_out) *n_cow_out = total_cow;
    return PKV_OK;
}

int pkv_seq_append_tables(pkv_alloc *a, const int64_t *seq_ids, int n, int n_tokens,
                          int64_t *slots_out, int32_t *cow_pairs_out, int *n_cow_out,
                          int *n_done_out, int32_t *tables_out, int32_t *lens_out) {
    if (n_done_out) *n_done_out = 0;
    if (n_cow_out) *n_cow_out = 0;
    if (n > 0 && !tables_out) return PKV_ERR_INVALID_ARG;
    const int rc = pkv_seq_append_batch(a, seq_ids, n, n_tokens, slots_out, cow_pairs_out,
                                        n_cow_out, n_done_out);
    if (rc != PKV_OK) return rc;
    return pkv_block_tables(a, seq_ids, n, tables_out, lens_out);
}

int pkv_seq_fork(pkv_alloc *a, int64_t parent, int64_t child) {
    return guarded([&]() -> int {
        if (!a) return PKV_ERR_INVALID_ARG;
        auto it = a->index.find(parent);
        if (it == a->index.end()) return PKV_ERR_UNKNOWN_SEQ;
        if (a->index.count(child)) return PKV_ERR_SEQ_EXISTS;
        const int32_t from = it->second;
        const int32_t to = a->add(child);
        const Seq &p = a->pool[from];
        Seq &c = a->pool[to];
        c.table.assign(p.table.begin(), p.table.end());
        c.len = p.len;
        c.tracked = p.tracked;
        c.hash = p.hash;
        c.partial.assign(p.partial.begin(), p.partial.end());
        for (int32_t b : c.table) a->refcount[b] += 1;
        a->logical_tokens += c.len;
        return PKV_OK;
    });
}

int pkv_seq_fork_batch(pkv_alloc *a, const int64_t *parents, const int64_t *children, int n,
                       int *n_done_out) {
    if (n_done_out) *n_done_out = 0;
    if (!a || n < 0 || (n > 0 && (!parents || !children))) return PKV_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        const int rc = pkv_seq_fork(a, parents[i], children[i]);
        if (rc != PKV_OK) return rc;
        if (n_done_out) *n_done_out = i + 1;
    }
    return PKV_OK;
}

int pkv_seq_free_batch(pkv_alloc *a, const int64_t *seq_ids, int n, int *n_done_out) {
    if (n_done_out) *n_done_out = 0;
    if (!a || n < 0 || (n > 0 && !seq_ids)) return PKV_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        const int rc = pkv_seq_free(a, seq_ids[i]);
        if (rc != PKV_OK) return rc;
        if (n_done_out) *n_done_out = i + 1;
    }
    return PKV_OK;
}

int pkv_seq_free(pkv_alloc *a, int64_t seq_id) {
    return guarded([&]() -> int {
        if (!a) return PKV_ERR_INVALID_ARG;
        auto it = a->index.find(seq_id);
        if (it == a->index.end()) return PKV_ERR_UNKNOWN_SEQ;
        const int32_t slot = it->second;
        Seq &s = a->pool[slot];
        for (auto b = s.table.rbegin(); b != s.table.rend(); ++b) {
            a->release(*b);
        }
        a->logical_tokens -= s.len;
        s.table.clear();
        s.partial.clear();
        a->index.erase(it);
        a->free_slots.push_back(slot);
        return PKV_OK;
    });
}

int pkv_block_tables(const pkv_alloc *a, const int64_t *seq_ids, int n, int32_t *tables_out,
                     int32_t *lens_out) {
    if (!a || n < 0 || (n > 0 && (!seq_ids || !tables_out))) return PKV_ERR_INVALID_ARG;
    const int mb = a->max_blocks;
    for (int i = 0; i < n; ++i) {
        const Seq *sp = a->find(seq_ids[i]);
        if (!sp) return PKV_ERR_UNKNOWN_SEQ;
        const Seq &s = *sp;
        int32_t *row = tables_out + (size_t)i * mb;
        const int k = (int)s.table.size();
        std::memcpy(row, s.table.data(), sizeof(int32_t) * k);
        std::fill(row + k, row + mb, -1);
        if (lens_out) lens_out[i] = (int32_t)s.len;
    }
    return PKV_OK;
}

int pkv_prefix_groups(const pkv_alloc *a, const int64_t *seq_ids, int n, int64_t *order_out,
                      int32_t *group_start_out, int32_t *prefix_lens_out, int *num_groups_out) {
    return guarded([&]() -> int {
        if (!a || n < 0 || !num_groups_out ||
            (n > 0 && (!seq_ids || !order_out || !group_start_out || !prefix_lens_out)))
            return PKV_ERR_INVALID_ARG;
        *num_groups_out = 0;
        if (n == 0) {
            if (group_start_out) group_start_out[0] = 0;
            return PKV_OK;
        }
        const int bs = a->block_size;
        std::vector<const Seq *> seqs(n);
        std::unordered_map<int64_t, int> seen;
        seen.reserve((size_t)n * 2);
        for (int i = 0; i < n; ++i) {
            seqs[i] = a->find(seq_ids[i]);
            if (!seqs[i]) return PKV_ERR_UNKNOWN_SEQ;
            if (!seen.emplace(seq_ids[i], i).second) return PKV_ERR_INVALID_ARG;   // repeated
        }
        // key: the physical block holding a sequence's first full block; none (own group)
        // for a sequence without a full block
        std::unordered_map<int32_t, int> group_of_block;
        std::vector<std::vector<int>> groups;
        for (int i = 0; i < n; ++i) {
            const Seq &s = *seqs[i];
            if (s.len >= bs && !s.table.empty()) {
                auto it = group_of_block.find(s.table[0]);
                if (it != group_of_block.end()) {
                    groups[it->second].push_back(i);
                    continue;
                }
                group_of_block.emplace(s.table[0], (int)groups.size());
            }
            groups.push_back({i});
        }
        int at = 0;
        for (size_t g = 0; g < groups.size(); ++g) {
            const std::vector<int> &m = groups[g];
            group_start_out[g] = at;
            int64_t common = 0;   // leading blocks every member holds, full in each
            if (m.size() > 1) {
                common = INT64_MAX;
                for (int i : m) common = std::min<int64_t>(common, seqs[i]->len / bs);
                const std::vector<int32_t> &t0 = seqs[m[0]]->table;
                for (size_t k = 1; k < m.size(); ++k) {
                    const std::vector<int32_t> &t = seqs[m[k]]->table;
                    int64_t b = 0;
                    while (b < common && t[(size_t)b] == t0[(size_t)b]) ++b;
                    common = b;
                }
            }
            prefix_lens_out[g] = (int32_t)std::min<int64_t>(common * bs, INT32_MAX);
            for (int i : m) order_out[at++] = seq_ids[i];
        }
        group_start_out[groups.size()] = at;
        *num_groups_out = (int)groups.size();
        return PKV_OK;
    });
}

int pkv_alloc_free_list(const pkv_alloc *a, int32_t *blocks_out, int max_out, int *n_out) {
    if (!a || !n_out || max_out < 0 || (max_out > 0 && !blocks_out)) return PKV_ERR_INVALID_ARG;
    int n = 0;
    for (auto it = a->free_stack.rbegin(); it != a->free_stack.rend() && n < max_out; ++it)
        blocks_out[n++] = *it;
    for (auto it = a->evictable.begin(); it != a->evictable.end() && n < max_out; ++it)
        blocks_out[n++] = *it;
    *n_out = n;
    return PKV_OK;
}

int pkv_alloc_refcounts(const pkv_alloc *a, int32_t *refcounts_out, int n) {
    if (!a || !refcounts_out || n < a->num_blocks) return PKV_ERR_INVALID_ARG;
    std::copy(a->refcount.begin(), a->refcount.end(), refcounts_out);
    return PKV_OK;
}

int pkv_stats(const pkv_alloc *a, int *free_blocks, int *held_blocks, int64_t *logical_tokens,
              double *utilisation) {
    if (!a) return PKV_ERR_INVALID_ARG;
    const int fr = a->available();
    const int held = a->num_blocks - fr;
    if (free_blocks) *free_blocks = fr;
    if (held_blocks) *held_blocks = held;
    if (logical_tokens) *logical_tokens = a->logical_tokens;
    if (utilisation)
        *utilisation = held ? (double)a->logical_tokens / ((double)held * a->block_size) : 0.0;
    return PKV_OK;
}

}  // extern "C"
