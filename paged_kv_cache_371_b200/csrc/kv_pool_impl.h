// Internal layout of the host block pool (opaque to callers as kv_pool*).
#pragma once

#include <cstdint>
#include <set>
#include <unordered_map>
#include <utility>
#include <vector>

#include "../../include/paged_kv.h"

struct kv_pool {
    kv_pool_config cfg;
    std::vector<int32_t> refcount;    // 0 = free
    std::vector<int32_t> free_stack;  // top = back()

    // Prefix cache (content-addressed full blocks).  Per block: whether it is
    // cached, the parent block named in its key, the number of cached
    // children, the tick of its last use; its tokens live in key_tokens
    // [block * block_size, +block_size).
    std::vector<uint8_t> cached;
    std::vector<int32_t> parent;
    std::vector<int32_t> children;
    std::vector<uint64_t> last_use;
    std::vector<int32_t> key_tokens;
    std::unordered_multimap<uint64_t, int32_t> by_hash;  // key hash -> block
    // (last use, block) of exactly the cached blocks that eviction may take:
    // no cached children and no reference but the cache's own
    std::set<std::pair<uint64_t, int32_t>> evictable;
    uint64_t clock = 0;
    int32_t n_cached = 0;
};

// Brings block b's membership of `evictable` up to date; called after any
// change to its reference count (a no-op while nothing was ever cached).
void kv_cache_recheck(kv_pool* p, int32_t b);
