// Content-addressed prefix cache over the host block pool.
//
// Follows "LLM 推理优化：KV Cache、PagedAttention 与量化" §2.3 (3): requests
// whose prompts share a prefix are detected by hashing block contents and
// point their block tables at the same physical blocks; and §2.3 (1): the pool
// keeps blocks nothing references in least-recently-used order.
//
// A cached block is identified by (parent, tokens): the cached block holding
// the previous block_size tokens (-1 for the first block) and its own
// block_size token ids, compared exactly.  Chaining the parent makes a match
// of block i imply a match of every earlier block, as the K/V rows of a block
// depend on all earlier tokens.  FNV-1a (64 bit) of the key only picks the
// bucket.  The cache holds one reference on every cached block.
#include <algorithm>
#include <cstdint>
#include <cstring>

#include "../../include/paged_kv.h"
#include "kv_pool_impl.h"
#include "kv_status.h"

namespace {

// FNV-1a 64 over the little-endian bytes of the parent id, then of the tokens.
uint64_t key_hash(int32_t parent, const int32_t* tokens, int32_t n)
{
    uint64_t h = 14695981039346656037ull;
    auto eat = [&h](int32_t v) {
        const uint32_t u = static_cast<uint32_t>(v);
        for (int i = 0; i < 4; ++i) {
            h ^= (u >> (8 * i)) & 0xffu;
            h *= 1099511628211ull;
        }
    };
    eat(parent);
    for (int32_t i = 0; i < n; ++i) eat(tokens[i]);
    return h;
}

bool ensure_cache(kv_pool* p)
{
    if (!p->cached.empty()) return true;
    const size_t n = static_cast<size_t>(p->cfg.num_blocks);
    const size_t bs = static_cast<size_t>(p->cfg.block_size);
    try {
        p->cached.assign(n, 0);
        p->parent.assign(n, -1);
        p->children.assign(n, 0);
        p->last_use.assign(n, 0);
        p->key_tokens.assign(n * bs, 0);
        p->by_hash.reserve(n);
    } catch (...) {
        p->cached.clear();
        return false;
    }
    return true;
}

// Cached block with exactly this key, or -1.
int32_t find(const kv_pool* p, uint64_t h, int32_t parent, const int32_t* tokens)
{
    const size_t bs = static_cast<size_t>(p->cfg.block_size);
    const auto range = p->by_hash.equal_range(h);
    for (auto it = range.first; it != range.second; ++it) {
        const int32_t b = it->second;
        if (p->parent[b] == parent &&
            std::memcmp(&p->key_tokens[static_cast<size_t>(b) * bs], tokens, bs * sizeof(int32_t)) == 0)
            return b;
    }
    return -1;
}

// Mark a block (cached, or about to be) as the most recently used.
void use(kv_pool* p, int32_t b)
{
    if (p->cached[b]) p->evictable.erase({p->last_use[b], b});
    p->last_use[b] = ++p->clock;
    kv_cache_recheck(p, b);
}

void uncache(kv_pool* p, int32_t b)
{
    const int32_t bs = p->cfg.block_size;
    p->evictable.erase({p->last_use[b], b});
    const uint64_t h = key_hash(p->parent[b], &p->key_tokens[static_cast<size_t>(b) * bs], bs);
    const auto range = p->by_hash.equal_range(h);
    for (auto it = range.first; it != range.second; ++it)
        if (it->second == b) {
            p->by_hash.erase(it);
            break;
        }
    const int32_t up = p->parent[b];
    if (up >= 0) --p->children[up];
    p->cached[b] = 0;
    p->parent[b] = -1;
    --p->n_cached;
    if (up >= 0) kv_cache_recheck(p, up);  // it may have become a leaf
}

}  // namespace

void kv_cache_recheck(kv_pool* p, int32_t b)
{
    if (p->cached.empty() || b < 0) return;
    const std::pair<uint64_t, int32_t> k{p->last_use[b], b};
    if (p->cached[b] && p->children[b] == 0 && p->refcount[b] == 1)
        p->evictable.insert(k);
    else
        p->evictable.erase(k);
}

extern "C" {

int kv_prefix_match(kv_pool* pool, const int32_t* tokens, int32_t n_tokens, int32_t* table_out,
                    int32_t table_capacity, int32_t* n_matched_out)
{
    if (!pool || !n_matched_out || n_tokens < 0 || (n_tokens > 0 && !tokens) || table_capacity < 0 ||
        (table_capacity > 0 && !table_out))
        return kv_fail(KV_ERR_INVALID, "kv_prefix_match: bad argument");
    *n_matched_out = 0;
    if (pool->cached.empty()) return KV_OK;  // nothing was ever cached
    const int32_t bs = pool->cfg.block_size;
    int32_t parent = -1, n = 0;
    for (int32_t i = 0; i < n_tokens / bs && n < table_capacity; ++i) {
        const int32_t* t = tokens + static_cast<size_t>(i) * bs;
        const int32_t b = find(pool, key_hash(parent, t, bs), parent, t);
        if (b < 0) break;
        ++pool->refcount[b];  // the new request's reference
        use(pool, b);
        table_out[n++] = b;
        parent = b;
    }
    *n_matched_out = n;
    return KV_OK;
}

int kv_prefix_register(kv_pool* pool, const int32_t* tokens, int32_t n_tokens, const int32_t* table,
                       int32_t n_blocks, int32_t* n_cached_out)
{
    if (!pool || n_tokens < 0 || n_blocks < 0 || (n_tokens > 0 && !tokens) || (n_blocks > 0 && !table))
        return kv_fail(KV_ERR_INVALID, "kv_prefix_register: bad argument");
    const int32_t bs = pool->cfg.block_size;
    const int32_t n = std::min(n_tokens / bs, n_blocks);
    for (int32_t i = 0; i < n; ++i)
        if (table[i] < 0 || table[i] >= pool->cfg.num_blocks || pool->refcount[table[i]] == 0)
            return kv_fail(KV_ERR_INVALID, "kv_prefix_register: table holds a block that is not live");
    if (n > 0 && !ensure_cache(pool)) return kv_fail(KV_ERR_OOM, "kv_prefix_register: out of host memory");
    int32_t parent = -1, done = 0;
    for (int32_t i = 0; i < n; ++i) {
        const int32_t b = table[i];
        const int32_t* t = tokens + static_cast<size_t>(i) * bs;
        const uint64_t h = key_hash(parent, t, bs);
        const int32_t have = find(pool, h, parent, t);
        if (have < 0) {
            if (pool->cached[b]) break;  // cached under another key
            pool->parent[b] = parent;
            std::memcpy(&pool->key_tokens[static_cast<size_t>(b) * bs], t, bs * sizeof(int32_t));
            pool->children[b] = 0;
            if (parent >= 0) ++pool->children[parent];
            pool->by_hash.emplace(h, b);
            ++pool->refcount[b];  // the cache's reference
            use(pool, b);
            pool->cached[b] = 1;
            ++pool->n_cached;
            kv_cache_recheck(pool, b);
            if (parent >= 0) kv_cache_recheck(pool, parent);  // no longer a leaf
        } else if (have == b) {
            use(pool, b);
        } else {
            break;  // this content is cached in another block
        }
        parent = b;
        ++done;
    }
    if (n_cached_out) *n_cached_out = done;
    return KV_OK;
}

int kv_prefix_evict(kv_pool* pool, int32_t n, int32_t* ids_out, int32_t* n_evicted_out)
{
    if (!pool || n < 0 || !n_evicted_out) return kv_fail(KV_ERR_INVALID, "kv_prefix_evict: bad argument");
    *n_evicted_out = 0;
    if (pool->cached.empty()) return KV_OK;
    int32_t k = 0;
    // the least recently used unreferenced leaf, each time: freeing a leaf
    // can make its parent one
    while (k < n && !pool->evictable.empty()) {
        const int32_t victim = pool->evictable.begin()->second;
        uncache(pool, victim);
        pool->refcount[victim] = 0;
        pool->free_stack.push_back(victim);
        if (ids_out) ids_out[k] = victim;
        ++k;
    }
    *n_evicted_out = k;
    return KV_OK;
}

int kv_prefix_num_cached(const kv_pool* pool, int32_t* n_out)
{
    if (!pool || !n_out) return kv_fail(KV_ERR_INVALID, "kv_prefix_num_cached: bad argument");
    *n_out = pool->n_cached;
    return KV_OK;
}

}  // extern "C"
