// Host block pool: free list, reference counts and the copy-on-write decision
// for paged KV caches. Pure host code; the device copy itself is
// pa_copy_blocks.
//
// Rules ([P2 "PagedAttention原理与KV Cache显存优化", §3.3-§3.4 and §4.2];
// [P4 "PagedAttention 实现细节", §3.3]; [P1 "PagedAttention 源码解析", §3]):
//   * allocate takes a block from the free list and sets its count to 1;
//     free drops the count and returns the block to the free list at 0;
//   * token t of a sequence goes to table[t / bs] at offset t % bs; a new
//     block is taken when t % bs == 0;
//   * before writing into a block whose count is above 1, take a new block,
//     record (old, new) for the device copy, drop the old block's count and
//     repoint the table; a block with count 1 is written in place.
#include <algorithm>
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa.h"

struct pa_block_pool {
    int num_blocks;
    int block_size;
    int policy;
    std::deque<int32_t> free_list;  // FIFO takes front, LIFO takes back; frees go to the back
    std::vector<int32_t> ref;

    bool valid(int b) const { return b >= 0 && b < num_blocks; }

    int take(int32_t *out) {
        if (free_list.empty()) return PA_ERR_POOL_EXHAUSTED;
        int32_t b;
        if (policy == PA_POOL_FIFO) {
            b = free_list.front();
            free_list.pop_front();
        } else {
            b = free_list.back();
            free_list.pop_back();
        }
        ref[b] = 1;
        *out = b;
        return PA_OK;
    }

    int drop(int b) {
        if (!valid(b) || ref[b] <= 0) return PA_ERR_POOL_STATE;
        if (--ref[b] == 0) free_list.push_back(b);
        return PA_OK;
    }
};

extern "C" {

pa_block_pool *pa_pool_create(int num_blocks, int block_size, int policy,
                              const int32_t *free_order) {
    if (num_blocks < 0 || block_size <= 0 || (policy != PA_POOL_LIFO && policy != PA_POOL_FIFO))
        return nullptr;
    pa_block_pool *p = new (std::nothrow) pa_block_pool();
    if (!p) return nullptr;
    p->num_blocks = num_blocks;
    p->block_size = block_size;
    p->policy = policy;
    p->ref.assign(num_blocks, 0);
    if (free_order) {
        std::vector<char> seen(num_blocks, 0);
        for (int i = 0; i < num_blocks; ++i) {
            const int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete p;
                return nullptr;
            }
            seen[b] = 1;
            p->free_list.push_back(b);
        }
    } else {
        for (int i = 0; i < num_blocks; ++i) p->free_list.push_back(i);
    }
    return p;
}

void pa_pool_destroy(pa_block_pool *pool) { delete pool; }

int pa_pool_num_free(const pa_block_pool *pool) {
    return pool ? (int)pool->free_list.size() : PA_ERR_NULL;
}

int pa_pool_ref_count(const pa_block_pool *pool, int block) {
    if (!pool) return PA_ERR_NULL;
    if (!pool->valid(block)) return PA_ERR_POOL_STATE;
    return pool->ref[block];
}

int pa_pool_allocate(pa_block_pool *pool, int32_t *block_out) {
    if (!pool || !block_out) return PA_ERR_NULL;
    return pool->take(block_out);
}

int pa_pool_share(pa_block_pool *pool, int block) {
    if (!pool) return PA_ERR_NULL;
    if (!pool->valid(block) || pool->ref[block] <= 0) return PA_ERR_POOL_STATE;
    ++pool->ref[block];
    return PA_OK;
}

int pa_pool_free(pa_block_pool *pool, int block) {
    if (!pool) return PA_ERR_NULL;
    return pool->drop(block);
}

int pa_pool_append(pa_block_pool *pool, int32_t *table, int max_blocks, int32_t *num_tokens,
                   int n_new, int32_t *slots, int64_t *cow_pairs, int cow_capacity, int *num_cow) {
    if (!pool || !table || !num_tokens || !num_cow) return PA_ERR_NULL;
    if (n_new < 0 || max_blocks < 0 || *num_tokens < 0 || cow_capacity < 0) return PA_ERR_SHAPE;
    if (cow_capacity > 0 && !cow_pairs) return PA_ERR_NULL;
    const int bs = pool->block_size;
    *num_cow = 0;
    for (int i = 0; i < n_new; ++i) {
        const int32_t t = *num_tokens;
        const int lb = t / bs;
        if (lb >= max_blocks) return PA_ERR_CAPACITY;
        if (t % bs == 0) {
            int32_t b;
            const int rc = pool->take(&b);
            if (rc != PA_OK) return rc;
            table[lb] = b;
        } else {
            const int32_t old = table[lb];
            if (!pool->valid(old) || pool->ref[old] <= 0) return PA_ERR_POOL_STATE;
            if (pool->ref[old] > 1) {
                if (*num_cow >= cow_capacity) return PA_ERR_CAPACITY;
                int32_t b;
                const int rc = pool->take(&b);
                if (rc != PA_OK) return rc;
                cow_pairs[2 * *num_cow] = old;
                cow_pairs[2 * *num_cow + 1] = b;
                ++*num_cow;
                pool->drop(old);
                table[lb] = b;
            }
        }
        if (slots) slots[i] = table[lb] * bs + t % bs;
        *num_tokens = t + 1;
    }
    return PA_OK;
}

int pa_pool_fork(pa_block_pool *pool, const int32_t *table, int num_tokens, int32_t *dst_table,
                 int max_blocks) {
    if (!pool || !table || !dst_table) return PA_ERR_NULL;
    if (num_tokens < 0) return PA_ERR_SHAPE;
    const int nb = (num_tokens + pool->block_size - 1) / pool->block_size;
    if (nb > max_blocks) return PA_ERR_CAPACITY;
    for (int j = 0; j < nb; ++j)
        if (!pool->valid(table[j]) || pool->ref[table[j]] <= 0) return PA_ERR_POOL_STATE;
    for (int j = 0; j < nb; ++j) {
        ++pool->ref[table[j]];
        dst_table[j] = table[j];
    }
    return PA_OK;
}

int pa_pool_export(const pa_block_pool *pool, int32_t *ref_counts, int32_t *free_list, int *num_free) {
    if (!pool || !ref_counts || !free_list || !num_free) return PA_ERR_NULL;
    std::copy(pool->ref.begin(), pool->ref.end(), ref_counts);
    std::copy(pool->free_list.begin(), pool->free_list.end(), free_list);
    *num_free = (int)pool->free_list.size();
    return PA_OK;
}

int pa_pool_release(pa_block_pool *pool, const int32_t *table, int num_tokens) {
    if (!pool || !table) return PA_ERR_NULL;
    if (num_tokens < 0) return PA_ERR_SHAPE;
    const int nb = (num_tokens + pool->block_size - 1) / pool->block_size;
    for (int j = 0; j < nb; ++j)
        if (!pool->valid(table[j]) || pool->ref[table[j]] <= 0) return PA_ERR_POOL_STATE;
    for (int j = 0; j < nb; ++j) pool->drop(table[j]);
    return PA_OK;
}

}  // extern "C"

// ------------------------------------------------------------ prefix cache
//
// [P4 "PagedAttention 实现细节", §3.2]: a prompt prefix (a system prompt) is
// computed once and its blocks are reused by every request that starts with
// it. get_or_create: a cached prompt's use count goes up and its blocks are
// returned; an unseen prompt gets ceil(len / bs) fresh blocks (all or none)
// and use count 1. release: the count drops and at zero the blocks go back
// to the pool and the entry is removed; an unknown prompt is ignored.
//
// Entries are bucketed by a 64-bit FNV-1a hash of the token ids (the
// published FNV-1a definition: offset basis 14695981039346656037, prime
// 1099511628211, over the ids' little-endian bytes), keeping the low
// hash_bits bits, and a hit also requires equal token lists: two prompts
// whose hashes agree never share blocks.

struct pa_prefix_cache {
    struct Entry {
        std::vector<int32_t> tokens;
        std::vector<int32_t> blocks;
        int ref_count;
    };
    pa_block_pool *pool;
    uint64_t mask;
    std::unordered_map<uint64_t, std::vector<Entry>> buckets;
    int entries = 0;

    uint64_t key(const int32_t *t, int n) const {
        uint64_t h = 14695981039346656037ull;
        for (int i = 0; i < n; ++i) {
            const uint32_t v = (uint32_t)t[i];
            for (int b = 0; b < 4; ++b) {
                h ^= (v >> (8 * b)) & 0xffu;
                h *= 1099511628211ull;
            }
        }
        return h & mask;
    }

    // The entry for this token list, or null; *bucket receives its bucket.
    Entry *find(const int32_t *t, int n, std::vector<Entry> **bucket) {
        auto it = buckets.find(key(t, n));
        if (it == buckets.end()) {
            *bucket = nullptr;
            return nullptr;
        }
        *bucket = &it->second;
        for (Entry &e : it->second)
            if ((int)e.tokens.size() == n && std::equal(e.tokens.begin(), e.tokens.end(), t)) return &e;
        return nullptr;
    }
};

extern "C" {

pa_prefix_cache *pa_prefix_cache_create(pa_block_pool *pool, int hash_bits) {
    if (!pool || hash_bits < 0 || hash_bits > 64) return nullptr;
    pa_prefix_cache *c = new (std::nothrow) pa_prefix_cache();
    if (!c) return nullptr;
    c->pool = pool;
    c->mask = (hash_bits == 0 || hash_bits == 64) ? ~0ull : ((1ull << hash_bits) - 1);
    return c;
}

void pa_prefix_cache_destroy(pa_prefix_cache *cache) { delete cache; }

int pa_prefix_num_entries(const pa_prefix_cache *cache) { return cache ? cache->entries : PA_ERR_NULL; }

int pa_prefix_get_or_create(pa_prefix_cache *cache, const int32_t *tokens, int num_tokens, int32_t *block_ids,
                            int max_blocks, int *num_ids, int *hit) {
    if (!cache || !num_ids || !hit || (num_tokens > 0 && !tokens)) return PA_ERR_NULL;
    if (num_tokens < 0 || max_blocks < 0) return PA_ERR_SHAPE;
    pa_block_pool *pool = cache->pool;
    const int nb = (num_tokens + pool->block_size - 1) / pool->block_size;
    if (nb > max_blocks) return PA_ERR_CAPACITY;
    if (nb > 0 && !block_ids) return PA_ERR_NULL;
    std::vector<pa_prefix_cache::Entry> *bucket = nullptr;
    pa_prefix_cache::Entry *e = cache->find(tokens, num_tokens, &bucket);
    if (e) {
        ++e->ref_count;
        std::copy(e->blocks.begin(), e->blocks.end(), block_ids);
        *num_ids = nb;
        *hit = 1;
        return PA_OK;
    }
    if ((int)pool->free_list.size() < nb) return PA_ERR_POOL_EXHAUSTED;
    pa_prefix_cache::Entry ne;
    ne.tokens.assign(tokens, tokens + num_tokens);
    ne.blocks.resize(nb);
    for (int j = 0; j < nb; ++j) pool->take(&ne.blocks[j]);
    ne.ref_count = 1;
    std::copy(ne.blocks.begin(), ne.blocks.end(), block_ids);
    if (!bucket) bucket = &cache->buckets[cache->key(tokens, num_tokens)];
    bucket->push_back(std::move(ne));
    ++cache->entries;
    *num_ids = nb;
    *hit = 0;
    return PA_OK;
}

int pa_prefix_release(pa_prefix_cache *cache, const int32_t *tokens, int num_tokens) {
    if (!cache || (num_tokens > 0 && !tokens)) return PA_ERR_NULL;
    if (num_tokens < 0) return PA_ERR_SHAPE;
    std::vector<pa_prefix_cache::Entry> *bucket = nullptr;
    pa_prefix_cache::Entry *e = cache->find(tokens, num_tokens, &bucket);
    if (!e) return PA_OK;
    if (e->ref_count == 1)  // the blocks go back: each must still be held
        for (int32_t b : e->blocks)
            if (!cache->pool->valid(b) || cache->pool->ref[b] <= 0) return PA_ERR_POOL_STATE;
    if (--e->ref_count > 0) return PA_OK;
    for (int32_t b : e->blocks) cache->pool->drop(b);
    bucket->erase(bucket->begin() + (e - bucket->data()));
    if (bucket->empty()) cache->buckets.erase(cache->key(tokens, num_tokens));
    --cache->entries;
    return PA_OK;
}

int pa_prefix_ref_count(pa_prefix_cache *cache, const int32_t *tokens, int num_tokens) {
    if (!cache || (num_tokens > 0 && !tokens)) return PA_ERR_NULL;
    if (num_tokens < 0) return PA_ERR_SHAPE;
    std::vector<pa_prefix_cache::Entry> *bucket = nullptr;
    const pa_prefix_cache::Entry *e = cache->find(tokens, num_tokens, &bucket);
    return e ? e->ref_count : 0;
}

}  // extern "C"
