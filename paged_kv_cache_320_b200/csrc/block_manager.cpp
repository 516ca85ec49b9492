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
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

namespace {

struct Seq {
    std::vector<int32_t> table;  // logical block -> physical block
    int64_t len = 0;             // tokens written
};

}  // namespace

struct pkv_alloc {
    int num_blocks = 0;
    int block_size = 0;
    int max_blocks = 0;
    std::vector<int32_t> free_stack;  // back() is the next block handed out
    std::vector<int32_t> refcount;
    std::unordered_map<int64_t, Seq> seqs;
    int64_t logical_tokens = 0;

    int32_t take() {
        int32_t b = free_stack.back();
        free_stack.pop_back();
        refcount[b] = 1;
        return b;
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
    pkv_alloc *a = new (std::nothrow) pkv_alloc();
    if (!a) return PKV_ERR_INVALID_ARG;
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->max_blocks = max_blocks_per_seq;
    a->refcount.assign(num_blocks, 0);
    a->free_stack.resize(num_blocks);
    for (int i = 0; i < num_blocks; ++i)
        a->free_stack[num_blocks - 1 - i] = initial_order ? initial_order[i] : i;
    *out = a;
    return PKV_OK;
}

int pkv_alloc_destroy(pkv_alloc *a) {
    delete a;
    return PKV_OK;
}

int pkv_seq_append(pkv_alloc *a, int64_t seq_id, int n_tokens, int64_t *slots_out,
                   int32_t *cow_pairs_out, int *n_cow_out) {
    if (!a || n_tokens < 0) return PKV_ERR_INVALID_ARG;
    if (n_tokens > 0 && !slots_out) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    const Seq *existing = it == a->seqs.end() ? nullptr : &it->second;
    int64_t need, table_len;
    a->needs(existing, n_tokens, &need, &table_len);
    if (table_len > a->max_blocks) return PKV_ERR_TABLE_FULL;
    if (need > (int64_t)a->free_stack.size()) return PKV_ERR_OUT_OF_BLOCKS;
    if (need > 0 && !cow_pairs_out && existing && existing->len % a->block_size != 0 &&
        a->refcount[existing->table.back()] > 1)
        return PKV_ERR_INVALID_ARG;  // a copy-on-write pair would be lost
    Seq &s = a->seqs[seq_id];
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
    }
    a->logical_tokens += n_tokens;
    if (n_cow_out) *n_cow_out = n_cow;
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

int pkv_seq_fork(pkv_alloc *a, int64_t parent, int64_t child) {
    if (!a) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(parent);
    if (it == a->seqs.end()) return PKV_ERR_UNKNOWN_SEQ;
    if (a->seqs.count(child)) return PKV_ERR_SEQ_EXISTS;
    Seq copy = it->second;
    for (int32_t b : copy.table) a->refcount[b] += 1;
    a->logical_tokens += copy.len;
    a->seqs.emplace(child, std::move(copy));
    return PKV_OK;
}

int pkv_seq_free(pkv_alloc *a, int64_t seq_id) {
    if (!a) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ERR_UNKNOWN_SEQ;
    const Seq &s = it->second;
    for (auto b = s.table.rbegin(); b != s.table.rend(); ++b) {
        if (--a->refcount[*b] == 0) a->free_stack.push_back(*b);
    }
    a->logical_tokens -= s.len;
    a->seqs.erase(it);
    return PKV_OK;
}

int pkv_block_tables(const pkv_alloc *a, const int64_t *seq_ids, int n, int32_t *tables_out,
                     int32_t *lens_out) {
    if (!a || n < 0 || (n > 0 && (!seq_ids || !tables_out))) return PKV_ERR_INVALID_ARG;
    const int mb = a->max_blocks;
    for (int i = 0; i < n; ++i) {
        auto it = a->seqs.find(seq_ids[i]);
        if (it == a->seqs.end()) return PKV_ERR_UNKNOWN_SEQ;
        const Seq &s = it->second;
        int32_t *row = tables_out + (size_t)i * mb;
        const int k = (int)s.table.size();
        std::memcpy(row, s.table.data(), sizeof(int32_t) * k);
        std::fill(row + k, row + mb, -1);
        if (lens_out) lens_out[i] = (int32_t)s.len;
    }
    return PKV_OK;
}

int pkv_stats(const pkv_alloc *a, int *free_blocks, int *held_blocks, int64_t *logical_tokens,
              double *utilisation) {
    if (!a) return PKV_ERR_INVALID_ARG;
    const int fr = (int)a->free_stack.size();
    const int held = a->num_blocks - fr;
    if (free_blocks) *free_blocks = fr;
    if (held_blocks) *held_blocks = held;
    if (logical_tokens) *logical_tokens = a->logical_tokens;
    if (utilisation)
        *utilisation = held ? (double)a->logical_tokens / ((double)held * a->block_size) : 0.0;
    return PKV_OK;
}

}  // extern "C"
